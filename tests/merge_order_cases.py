"""Order-sensitive merge cases shared by the oracle pins and the GPU parity tests.

Each builder returns the inputs of one operation whose row (token 7 or 3, channel 0) merges
four candidates into one target, the candidates' fp32 weights in the pages-reading's order
(ascending candidate order), and the same weights in a plausible wrong order. The other
channels and tokens carry zero weights. `k` sets the channel count, so the GPU tests can place
the case where the tiled kernels run. The weights are three-decimal fp32 values (not dyadic)
whose ascending-order fp32 sum differs from the sum in every other order the tests name.
"""
import numpy as np

f32 = np.float32


def asc(vals):
    """fp32 sum in the given order, each add rounded once."""
    s = f32(vals[0])
    for v in vals[1:]:
        s = f32(s + f32(v))
    return s


# ---- SER: four two-hop paths to one target ---------------------------------------------------
#
# Row (token 7, channel 0) with first leg (5, 0.242), (6, 0.361); second-leg rows 5 and 6 point
# both slots at target 2. Candidates c = a*s3 + e: (0,0) (0,1) (1,0) (1,1).

SER_W1 = [f32("0.242"), f32("0.361")]
SER_W2 = [[f32("0.951"), f32("0.777")], [f32("0.331"), f32("0.935")]]


def ser_case(k=1, n=8):
    s = 2
    a1_idx = np.zeros((1, n, k, s), np.int32)
    a1_w = np.zeros((1, n, k, s), np.float32)
    a2_idx = np.zeros((1, n, k, s), np.int32)
    a2_w = np.zeros((1, n, k, s), np.float32)
    a1_idx[0, 7, 0] = [5, 6]
    a1_w[0, 7, 0] = SER_W1
    for a, j in enumerate((5, 6)):
        a2_idx[0, j, 0] = [2, 2]
        a2_w[0, j, 0] = SER_W2[a]
    u = [f32(SER_W1[a] * SER_W2[a][e]) for a in range(2) for e in range(2)]
    ut = [f32(SER_W1[a] * SER_W2[a][e]) for e in range(2) for a in range(2)]
    return (a1_idx, a1_w, a2_idx, a2_w), u, ut


# ---- referral with refresh edges: two paths, then two refresh slots, one target --------------

RF_W1 = [f32("0.733"), f32("0.851")]
RF_W2 = [f32("0.863"), f32("0.291")]
RF_F = [f32("0.732"), f32("0.133")]


def refresh_case(k=1, n=8, s3=1):
    """Paths (7 -> 4 -> 3) and (7 -> 5 -> 3), then refresh slots (3, 0.732), (3, 0.133).
    s3 > 1 pads the second leg with zero-weight slots."""
    a1_idx = np.zeros((1, n, k, 2), np.int32)
    a1_w = np.zeros((1, n, k, 2), np.float32)
    a2_idx = np.zeros((1, n, k, s3), np.int32)
    a2_w = np.zeros((1, n, k, s3), np.float32)
    f_idx = np.zeros((1, n, k, 2), np.int32)
    f_w = np.zeros((1, n, k, 2), np.float32)
    a1_idx[0, 7, 0] = [4, 5]
    a1_w[0, 7, 0] = RF_W1
    a2_idx[0, 4, 0, 0] = 3
    a2_w[0, 4, 0, 0] = RF_W2[0]
    a2_idx[0, 5, 0, 0] = 3
    a2_w[0, 5, 0, 0] = RF_W2[1]
    f_idx[0, 7, 0] = [3, 3]
    f_w[0, 7, 0] = RF_F
    p = [f32(RF_W1[a] * RF_W2[a]) for a in range(2)]
    return (a1_idx, a1_w, a2_idx, a2_w, f_idx, f_w), p + RF_F, RF_F + p


# ---- leg sparsification: two stored channels x two slots, one target --------------------------

LEG_M = [f32("0.803"), f32("0.784")]                    # M1[h=0, c] for c = 0, 1
LEG_EW = [[f32("0.295"), f32("0.637")], [f32("0.649"), f32("0.901")]]  # E.w[c, a]


def leg_case(k=2, n=4):
    """Token 3 stores (1, w) in slots (c, a) for c, a < 2; leg 1 of channel 0 mixes them with
    M1[0, :2]. Every other coefficient is 0.5, every other stored slot inactive."""
    s0 = 2
    e_idx = np.zeros((1, n, k, s0), np.int32)
    e_w = np.zeros((1, n, k, s0), np.float32)
    e_idx[0, 3, :2] = 1
    e_w[0, 3, :2] = LEG_EW
    mix1 = np.full((k, k), f32("0.5"), np.float32)
    mix1[0] = 0.0
    mix1[0, :2] = LEG_M
    mix2 = np.full((k, k), f32("0.5"), np.float32)
    u = [f32(LEG_M[c] * LEG_EW[c][a]) for c in range(2) for a in range(s0)]
    ut = [f32(LEG_M[c] * LEG_EW[c][a]) for a in range(s0) for c in range(2)]
    return (e_idx, e_w, mix1, mix2), u, ut
