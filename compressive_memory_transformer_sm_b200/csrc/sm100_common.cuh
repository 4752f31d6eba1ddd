// Shared pieces of the tensor-core (tcgen05 / TMEM / TMA) kernels of the
// Infini-attention forward for bf16 inputs with d_key = d_value = 128 on
// sm_100a: tile geometry, shared-memory matrix descriptors, swizzled chunk
// addressing.  The kernels are in sm100_attn.cuh and sm100_update.cuh.
//
// Operand tiles are 128 rows x 128 bf16 columns, held in shared memory as two
// TMA boxes of 128 rows x 64 columns (16 KB each) with the 128-byte swizzle:
// 16-byte chunk c of row r sits at chunk position c ^ (r % 8) of the row.
// A tile is K-major when its rows are the MMA's M/N index (Q, K, sigma(Q));
// it is MN-major when its rows are the MMA's K index (V, U, the memory
// snapshot M_{s-1} [dk][dv], sigma(K) read as sigma(K)^T).
#pragma once

#include "common.cuh"

namespace infini {
namespace tc {

constexpr int kTile = 128;
constexpr uint32_t kBox = 16384;        // 128 rows x 128 B
constexpr uint32_t kTileBytes = 32768;  // two boxes

// Descriptor of K-step kk (16 elements along K) of a K-major tile: the
// descriptor of step 0 plus the step's offset in the start-address field.
// Shared-memory addresses stay below 256 KB, so (address >> 4) fits the
// 14-bit field and the addition never carries out of it; the base is then
// computed once per tile and each step costs one add.
__device__ __forceinline__ uint64_t kmajor_base(uint32_t tile) { return smem_desc_sw128(tile, 16u, 1024u); }
__host__ __device__ constexpr uint64_t kmajor_step(int kk) {
  return (uint64_t)((uint32_t)(kk >> 2) * (kBox >> 4) + (uint32_t)(kk & 3) * 2u);
}
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t tile, int kk) { return kmajor_base(tile) + kmajor_step(kk); }
// Descriptor of K-step kk (16 rows along K) of an MN-major tile.
__device__ __forceinline__ uint64_t mnmajor_base(uint32_t tile) { return smem_desc_sw128(tile, kBox, 1024u); }
__host__ __device__ constexpr uint64_t mnmajor_step(int kk) { return (uint64_t)((uint32_t)kk * (2048u >> 4)); }
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t tile, int kk) { return mnmajor_base(tile) + mnmajor_step(kk); }
// Descriptor of K-step kk of the 16-row K-major block of ones (two 2 KB boxes).
__device__ __forceinline__ uint64_t ones_desc(uint32_t tile, int kk) {
  return smem_desc_sw128(tile + (uint32_t)(kk >> 2) * 2048u + (uint32_t)(kk & 3) * 32u, 16u, 1024u);
}
// Byte offset of 16-byte chunk c (0..15, 8 bf16 each) of row r inside a tile.
__device__ __forceinline__ uint32_t swz_chunk(int r, int c) {
  return (uint32_t)(c >> 3) * kBox + (uint32_t)r * 128u + ((uint32_t)((c & 7) ^ (r & 7)) << 4);
}

__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ void sts128(uint32_t a, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

}  // namespace tc
}  // namespace infini
