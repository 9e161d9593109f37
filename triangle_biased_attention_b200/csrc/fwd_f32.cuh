// Biased-attention forward with plain FMA arithmetic in fp32 throughout, for
// fp32 inputs and for the bf16 shapes the tensor-core kernel does not take.
//
// The same operation as the bf16 kernel (DeepSpeed DS4Sci_EvoformerAttention
// guide, hmyw.cn, sections 4, 5.2 and 5.4).  For fp32 inputs it is the whole
// path, because tensor-core TF32 would not hold a 1e-5 relative error; for
// bf16 inputs (T = raw bf16 bits) it serves any head dimension up to 128 and
// pair biases whose rows are not a multiple of 16 bytes, at SIMT speed, with
// O rounded to bf16 at the end.  One warp owns one query row;
// K and V blocks of 64 keys are staged in shared memory for the 8 rows of a
// CTA.  Each lane scores two keys of a block, the warp takes the block max
// and sum with xor-shuffles, then each lane accumulates its D/32 output
// columns.  The mask is rebased per (b, n) by its maximum, as in the bf16
// kernel, so an n whose every key carries -1e9 still follows the formula.
#pragma once

#include <cstdint>

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"

namespace evo {

constexpr int kF32Rows = 8;   // query rows (warps) per CTA
constexpr int kF32Keys = 64;  // keys per shared-memory block
constexpr int kF32MaxD = 128;

// Element access: fp32 as stored, bf16 as raw bits (exact widening; output
// rounded to nearest even).
__device__ __forceinline__ float ld_elem(const float* p, size_t i) { return p[i]; }
__device__ __forceinline__ float ld_elem(const uint16_t* p, size_t i) { return __uint_as_float(uint32_t(p[i]) << 16); }
__device__ __forceinline__ void st_elem(float* p, size_t i, float x) { p[i] = x; }
__device__ __forceinline__ void st_elem(uint16_t* p, size_t i, float x) {
    p[i] = __bfloat16_as_ushort(__float2bfloat16_rn(x));
}
// fp16 (exact widening; output rounded to nearest even)
__device__ __forceinline__ float ld_elem(const __half* p, size_t i) { return __half2float(p[i]); }
__device__ __forceinline__ void st_elem(__half* p, size_t i, float x) { p[i] = __float2half_rn(x); }

template <typename T>  // float, uint16_t holding bf16, or __half
struct F32Params {
    const T* q;
    const T* k;
    const T* v;
    const T* mask;  // [B, N, S] or nullptr
    const T* pair;  // [B, H, S, S] or nullptr
    T* out;
    float* lse;
    int N, S, H, D;
    int ld;             // padded smem row (D + 1)
    int num_qb;         // query blocks of kF32Rows per (b, n, h)
    float scale;        // 1 / sqrt(D)
};

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

template <typename T>
__global__ void __launch_bounds__(kF32Rows * 32) evo_fwd_f32_kernel(const F32Params<T> p) {
    extern __shared__ float fsm[];
    float* Ks = fsm;                           // [kF32Keys][ld]
    float* Vs = Ks + kF32Keys * p.ld;          // [kF32Keys][ld]
    float* Qs = Vs + kF32Keys * p.ld;          // [kF32Rows][ld]
    float* Ps = Qs + kF32Rows * p.ld;          // [kF32Rows][kF32Keys]
    float* red = Ps + kF32Rows * kF32Keys;     // [kF32Rows]

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    long long t = blockIdx.x;
    const int qb = int(t % p.num_qb);
    t /= p.num_qb;
    const int h = int(t % p.H);
    const long long bn = t / p.H;  // b * N + n
    const long long b = bn / p.N;
    const int row = qb * kF32Rows + warp;
    const int D = p.D;
    const size_t row_stride = size_t(p.H) * D;  // between consecutive s in [B,N,S,H,D]
    const size_t slice_base = size_t(bn) * p.S * row_stride + size_t(h) * D;

    // per-(b, n) mask rebase
    const T* mrow = p.mask ? p.mask + size_t(bn) * p.S : nullptr;
    float c = 0.f;
    if (mrow) {
        float mx = -INFINITY;
        for (int j = threadIdx.x; j < p.S; j += blockDim.x) mx = fmaxf(mx, ld_elem(mrow, j));
        mx = warp_max(mx);
        if (lane == 0) red[warp] = mx;
        __syncthreads();
        mx = red[0];
        for (int i = 1; i < kF32Rows; ++i) mx = fmaxf(mx, red[i]);
        c = (mx == -INFINITY) ? 0.f : mx;
    }
    const T* prow = (p.pair && row < p.S) ? p.pair + (size_t(b) * p.H + h) * size_t(p.S) * p.S + size_t(row) * p.S
                                           : nullptr;

    for (int d = lane; d < D; d += 32)
        Qs[warp * p.ld + d] = row < p.S ? ld_elem(p.q, slice_base + size_t(row) * row_stride + d) : 0.f;

    float m = -INFINITY, l = 0.f;
    float o[kF32MaxD / 32] = {0.f, 0.f, 0.f, 0.f};
    for (int kb = 0; kb < p.S; kb += kF32Keys) {
        __syncthreads();
        for (int i = threadIdx.x; i < kF32Keys * D; i += blockDim.x) {
            const int jj = i / D, d = i - jj * D;
            const int key = kb + jj;
            const size_t off = slice_base + size_t(key) * row_stride + d;
            Ks[jj * p.ld + d] = key < p.S ? ld_elem(p.k, off) : 0.f;
            Vs[jj * p.ld + d] = key < p.S ? ld_elem(p.v, off) : 0.f;
        }
        __syncthreads();
        float tj[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int jj = lane + 32 * e;
            const int key = kb + jj;
            float x = -INFINITY;
            if (key < p.S && row < p.S) {
                float dot = 0.f;
                for (int d = 0; d < D; ++d) dot = fmaf(Qs[warp * p.ld + d], Ks[jj * p.ld + d], dot);
                x = dot * p.scale;
                if (mrow) x += ld_elem(mrow, key) - c;
                if (prow) x += ld_elem(prow, key);
            }
            tj[e] = x;
        }
        const float m_new = fmaxf(m, warp_max(fmaxf(tj[0], tj[1])));
        const float m_safe = (m_new == -INFINITY) ? 0.f : m_new;
        const float alpha = (m == -INFINITY) ? 0.f : expf(m - m_safe);
        const float p0 = expf(tj[0] - m_safe);
        const float p1 = expf(tj[1] - m_safe);
        l = l * alpha + warp_sum(p0 + p1);
        Ps[warp * kF32Keys + lane] = p0;
        Ps[warp * kF32Keys + lane + 32] = p1;
        __syncwarp();
#pragma unroll
        for (int i = 0; i < kF32MaxD / 32; ++i) {
            const int d = lane + 32 * i;
            if (d < D) {
                float acc = o[i] * alpha;
                for (int jj = 0; jj < kF32Keys; ++jj) acc = fmaf(Ps[warp * kF32Keys + jj], Vs[jj * p.ld + d], acc);
                o[i] = acc;
            }
        }
        m = m_new;
        __syncwarp();
    }
    if (row < p.S) {
        const float inv_l = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
        for (int i = 0; i < kF32MaxD / 32; ++i) {
            const int d = lane + 32 * i;
            if (d < D) st_elem(p.out, slice_base + size_t(row) * row_stride + d, o[i] * inv_l);
        }
        if (lane == 0)
            p.lse[(size_t(bn) * p.H + h) * size_t(p.S) + row] = l > 0.f ? m + logf(l) + c : -INFINITY;
    }
}

}  // namespace evo
