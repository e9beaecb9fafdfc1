// Host-only cross-check of the tcgen05 descriptor encoders (csrc/umma.h) against the
// bitfield unions of CUTLASS's cute/arch/mma_sm100_desc.hpp (source headers).
#include <cstdio>
#include <cstdint>
#include <cute/arch/mma_sm100_desc.hpp>
#include "umma.h"

static int fails = 0;
#define CHECK(a, b) do { if ((a) != (b)) { std::printf("MISMATCH %s: %llx vs %llx\n", #a, \
    (unsigned long long)(a), (unsigned long long)(b)); ++fails; } } while (0)

int main() {
    // shared-memory descriptors: K-major SW128 (LBO 16, SBO 1024) and MN-major (LBO 16 KiB)
    const uint32_t addrs[] = {0x0, 0x400, 0x8020, 0x1C060, 0x3FC00};
    const uint32_t lbos[] = {16, 16384};
    for (uint32_t a : addrs) for (uint32_t lbo : lbos) {
        cute::UMMA::SmemDescriptor d;
        d.desc_ = 0;
        d.start_address_ = a >> 4;
        d.leading_byte_offset_ = lbo >> 4;
        d.stride_byte_offset_ = 1024 >> 4;
        d.version_ = 1;
        d.base_offset_ = 0;
        d.lbo_mode_ = 0;
        d.layout_type_ = uint8_t(cute::UMMA::LayoutType::SWIZZLE_128B);
        CHECK(swa::umma::smem_desc(a, lbo, 1024), d.desc_);
    }
    // instruction descriptors: S = Q K^T (128x128, K-major B) and O += P V (128xD, MN-major B)
    const uint32_t Ns[] = {64, 128};
    for (uint32_t n : Ns) for (uint32_t bmn = 0; bmn < 2; ++bmn) {
        cute::UMMA::InstrDescriptor i;
        i.desc_ = 0;
        i.c_format_ = uint8_t(cute::UMMA::CFormat::F32);
        i.a_format_ = uint8_t(cute::UMMA::F16F32Format::BF16);
        i.b_format_ = uint8_t(cute::UMMA::F16F32Format::BF16);
        i.a_major_ = 0;
        i.b_major_ = bmn;
        i.n_dim_ = n >> 3;
        i.m_dim_ = 128 >> 4;
        CHECK(swa::umma::idesc_bf16_f32(128, n, bmn), i.desc_);
    }
    std::printf(fails ? "FAIL\n" : "OK\n");
    return fails ? 1 : 0;
}
