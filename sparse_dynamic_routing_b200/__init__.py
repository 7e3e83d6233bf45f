"""Graph Machine sparse layer (SER + SEA) for NVIDIA B200 (sm_100a).

The compute lives in the CUDA library libgm_b200.so (C ABI: include/gm.h); this package is
its Python binding plus the seeded synthetic-input generators (`inputs`).

    gm_leg_sparsify     both referral legs from the stored edges (mixed, then sparsified)
    gm_leg_backward     gradients of the kept leg weights
    gm_ser_forward      sparse edge referral, A' = Sparsify_s1(A1 A2)
    gm_ser_chain_forward / _backward, gm_ser_sea_chain_forward
                        multi-step referral, B_{m+1} = Sparsify(B_m A_{m+1})
    gm_ser_refresh_forward / _backward, gm_ser_sea_refresh_forward
                        the referral with refresh edges, A' = Sparsify_s1(A1 A2 + F)
    gm_sea_forward      sparse edge attention
    gm_ser_sea_forward  both in one kernel
    gm_sea_backward     gradients of sparse edge attention
    gm_ser_backward     gradients of the kept referral weights
    gm_ser_sea_backward both backward passes in one call (the referral's inside the attention's)
    gm_dense_refresh_edges
                        refresh edges from a dense attention layer (its top positions)
    gm_selftest_wait_timeout
                        diagnostic: one bounded wait that runs out (GM_ERR_WAIT_TIMEOUT)
"""
from ._binding import (  # noqa: F401
    GM_BF16,
    GM_F32,
    GMEdgeInvalidError,
    GMError,
    GMIndexRangeError,
    CHECKED_LIB_PATH,
    LIB_PATH,
    gm_check_device_errors,
    gm_dense_refresh_edges,
    gm_leg_backward,
    gm_leg_sparsify,
    gm_sea_backward,
    gm_sea_backward_noalloc,
    gm_sea_backward_workspace_size,
    gm_sea_forward,
    gm_ser_backward,
    gm_ser_chain_backward,
    gm_ser_chain_forward,
    gm_ser_forward,
    gm_ser_refresh_backward,
    gm_ser_refresh_forward,
    gm_ser_sea_chain_forward,
    gm_ser_sea_refresh_forward,
    gm_ser_sea_backward,
    gm_ser_sea_forward,
    gm_selftest_wait_timeout,
    gm_version,
    load_library,
    status_string,
)
