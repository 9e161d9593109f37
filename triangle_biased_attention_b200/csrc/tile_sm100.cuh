// Shared pieces of the tcgen05 kernels: tile constants, shared-memory matrix
// descriptors for the tensor cores (the bit layout of the PTX ISA's
// tcgen05 shared-memory descriptor), the swizzle of TMA-written tiles, and the
// in-place bf16 -> fp16 conversion of V tiles.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "ptx_sm100.cuh"

namespace evo {

constexpr int kBM = 128;          // query rows per tile
constexpr int kBN = 128;          // keys per block
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
// Masks more than this far below a row's running mask maximum (natural-log
// units) are treated as -inf; see the mask-column writers.
constexpr float kMaskFloor = 16384.0f;

// UMMA shared-memory descriptor layout codes for swizzle spans of 32/64/128 B.
__host__ __device__ constexpr uint32_t umma_layout_code(int sw_bytes) {
    return sw_bytes == 128 ? 2u : (sw_bytes == 64 ? 4u : 6u);
}

// K-major operand tile: rows of ROW bytes, swizzled over ROW bytes, 8-row
// groups ROW*8 bytes apart.
template <int ROW>
__device__ __forceinline__ uint64_t desc_k_major(uint32_t saddr) {
    uint64_t d = 0;
    d |= uint64_t((saddr >> 4) & 0x3FFFu);
    d |= uint64_t(1) << 16;                                  // leading offset (unused here)
    d |= uint64_t(((8u * ROW) >> 4) & 0x3FFFu) << 32;        // stride between 8-row groups
    d |= uint64_t(1) << 46;                                  // descriptor version (sm_100)
    d |= uint64_t(umma_layout_code(ROW)) << 61;
    return d;
}

// MN-major operand (V as the B operand of P.V: N = head dim contiguous, K =
// keys along rows).  One swizzle atom spans ROW bytes of N; the next atom of N
// (the ones tile) is `atom_stride` bytes further; 8-key groups are ROW*8 apart.
template <int ROW>
__device__ __forceinline__ uint64_t desc_mn_major(uint32_t saddr, uint32_t atom_stride) {
    uint64_t d = 0;
    d |= uint64_t((saddr >> 4) & 0x3FFFu);
    d |= uint64_t((atom_stride >> 4) & 0x3FFFu) << 16;
    d |= uint64_t(((8u * ROW) >> 4) & 0x3FFFu) << 32;
    d |= uint64_t(1) << 46;
    d |= uint64_t(umma_layout_code(ROW)) << 61;
    return d;
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Byte offset of 16 B chunk c of row r in a tile of ROW-byte rows stored with
// the ROW-byte swizzle (the layout TMA writes and the MMA descriptors name):
// the chunk index is XORed with bits of the row's position in the 1024 B atom.
template <int ROW>
__device__ __forceinline__ uint32_t swz_chunk(int r, int c) {
    const int sw = ((r * ROW) >> 7) & (ROW / 16 - 1);
    return uint32_t(r * ROW) + uint32_t((c ^ sw) << 4);
}

// 16 B chunks FIRST .. FIRST + COUNT - 1 of every lane (chunk g of lane l is
// the tile's chunk l + 32 g) of a V tile, bf16 -> fp16 in place (same
// swizzled positions), by one warp; then the async-proxy fence that makes the
// generic writes visible to the tensor cores.
template <int FIRST, int COUNT, bool ROLLED = false>
__device__ __forceinline__ void convert_v_chunks(uint32_t tile, int lane) {
    static_assert(FIRST % 4 == 0 && COUNT % 4 == 0, "whole groups of four");
#pragma unroll(ROLLED ? 1 : COUNT / 4)
    for (int g = FIRST; g < FIRST + COUNT; g += 4) {
        uint4 vv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) vv[u] = ptx::ld_shared_v4(tile + uint32_t((lane + 32 * (g + u)) * 16));
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            uint4 o;
            o.x = ptx::pack_f16x2(ptx::bf16lo_to_f32(vv[u].x), ptx::bf16hi_to_f32(vv[u].x));
            o.y = ptx::pack_f16x2(ptx::bf16lo_to_f32(vv[u].y), ptx::bf16hi_to_f32(vv[u].y));
            o.z = ptx::pack_f16x2(ptx::bf16lo_to_f32(vv[u].z), ptx::bf16hi_to_f32(vv[u].z));
            o.w = ptx::pack_f16x2(ptx::bf16lo_to_f32(vv[u].w), ptx::bf16hi_to_f32(vv[u].w));
            ptx::st_shared_v4(tile + uint32_t((lane + 32 * (g + u)) * 16), o);
        }
    }
    ptx::fence_proxy_async_smem();  // generic-proxy writes -> tensor-core reads
    __syncwarp();
}

}  // namespace evo
