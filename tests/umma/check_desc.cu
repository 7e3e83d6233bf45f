// Host-only check of the tcgen05 descriptor encodings in gm_umma.cuh against CUTLASS's
// definitions of the same bit fields (cute/arch/mma_sm100_desc.hpp). Prints "ok" or the
// first mismatch. Built and run by tests/test_umma_desc.py; needs no GPU.
#include <cstdio>

#include <cute/arch/mma_sm100_desc.hpp>
#include <cute/numeric/numeric_types.hpp>

#include "../../sparse_dynamic_routing_b200/csrc/gm_umma.cuh"

int main()
{
    int bad = 0;
    for (int n : {16, 64, 128, 256}) {
        cute::UMMA::InstrDescriptor want{};
        want.c_format_ = uint8_t(cute::UMMA::CFormat::F32);
        want.a_format_ = uint8_t(cute::UMMA::F16F32Format::BF16);
        want.b_format_ = uint8_t(cute::UMMA::F16F32Format::BF16);
        want.a_major_ = uint8_t(cute::UMMA::Major::K);
        want.b_major_ = uint8_t(cute::UMMA::Major::K);
        want.m_dim_ = 128 >> 4;
        want.n_dim_ = n >> 3;
        const uint32_t got = gm::umma::idesc_bf16_f32(128, n);
        if (got != want.desc_) {
            std::printf("idesc N=%d: got %08x want %08x\n", n, got, want.desc_);
            ++bad;
        }
        // the CUTLASS builder agrees with the hand-set fields
        const auto built = cute::UMMA::make_instr_desc<cute::bfloat16_t, cute::bfloat16_t, float, 128, 128,
                                                       cute::UMMA::Major::K, cute::UMMA::Major::K>();
        if (n == 128 && built.desc_ != got) {
            std::printf("idesc builder: got %08x want %08x\n", got, built.desc_);
            ++bad;
        }
    }
    for (uint32_t addr : {0u, 1024u, 1024u + 32u, 65536u + 96u, 230000u & ~15u}) {
        cute::UMMA::SmemDescriptor want{};
        want.start_address_ = (uint16_t)(addr >> 4);
        want.leading_byte_offset_ = 1;
        want.stride_byte_offset_ = 1024 >> 4;
        want.version_ = 1;
        want.base_offset_ = 0;
        want.lbo_mode_ = 0;
        want.layout_type_ = uint8_t(cute::UMMA::LayoutType::SWIZZLE_128B);
        const uint64_t got = gm::umma::sdesc_sw128_kmajor(addr);
        if (got != want.desc_) {
            std::printf("sdesc addr=%u: got %016llx want %016llx\n", addr, (unsigned long long)got,
                        (unsigned long long)want.desc_);
            ++bad;
        }
    }
    std::printf(bad ? "FAIL\n" : "ok\n");
    return bad ? 1 : 0;
}
