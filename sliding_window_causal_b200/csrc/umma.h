// umma.h: encoders for the sm_100a tensor-core (tcgen05) operand descriptors.
//
// Shared-memory matrix descriptor (64 bits):
//   [0,14)  start address >> 4        [16,30) leading byte offset >> 4
//   [32,46) stride byte offset >> 4   [46,48) version, 1 on sm_100
//   [49,52) base offset (0: tiles are 1024-byte aligned)
//   [52]    leading-offset mode (0)   [61,64) layout: 2 = 128-byte swizzle
// Instruction descriptor for kind::f16 (32 bits):
//   [4,6) D format (1 = f32)  [7,10) A format (1 = bf16)  [10,13) B format (1 = bf16)
//   [15] A major (0 = K)  [16] B major (0 = K, 1 = MN)  [17,23) N >> 3  [24,29) M >> 4
//
// Operand tiles are written by TMA with 128-byte swizzle: a row of 64 bf16 values is
// 128 bytes, 8 rows form a 1024-byte swizzle atom, and a 128-row tile of 64 columns
// is 16 KiB. With K-major operands (Q and K tiles) one MMA step of K = 16 bf16 is a
// 32-byte slice of each row: the descriptor start moves by 32 bytes per step inside
// a 64-column block and by 16 KiB to the next block; SBO = 1024 (8 rows), LBO unused
// (encoded 1). The V tile is the MN-major B operand of O += P.V (keys are K, head
// dimension is N): one step of 16 keys moves the start by 16 rows = 2048 bytes;
// LBO = 16 KiB (next 64-column block along N), SBO = 1024 (next 8 keys).
#pragma once
#include <stdint.h>

#if defined(__CUDACC__)
#define SWA_UMMA_HD __host__ __device__ __forceinline__ constexpr
#else
#define SWA_UMMA_HD inline constexpr
#endif

namespace swa {
namespace umma {

constexpr uint32_t kLayoutSwizzle128B = 2;

SWA_UMMA_HD uint64_t smem_desc(uint32_t smem_addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    return (uint64_t)((smem_addr & 0x3FFFFu) >> 4) |
           ((uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32) |
           ((uint64_t)1 << 46) |
           ((uint64_t)kLayoutSwizzle128B << 61);
}

// bf16 x bf16 -> f32, M x N tile; b_mn_major selects an MN-major B operand.
SWA_UMMA_HD uint32_t idesc_bf16_f32(uint32_t M, uint32_t N, uint32_t b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (0u << 15) | ((b_mn_major & 1u) << 16) |
           ((N >> 3) << 17) | ((M >> 4) << 24);
}

}  // namespace umma
}  // namespace swa
