// Backward pass of biased attention with plain FMA arithmetic in fp32: the
// row-statistics kernels that every backward path runs first, and the SIMT
// gradient kernels used for fp32 inputs and for the head dimensions the
// tensor-core backward does not take.
//
// What is computed (the DeepSpeed DS4Sci_EvoformerAttention guide, hmyw.cn,
// sections 1 and 5.4: the backward pass returns the gradients of Q, K, V and,
// when asked for, of the two biases, recomputing the attention weights from
// Q, K, V, O and the forward's log-sum-exp rather than storing them, with the
// per-row delta as an intermediate).  The guide prints no formula; this is the
// chain rule of the forward formula.  Per (b, n, h) slice, with
// t_ij = q_i . k_j / sqrt(D) + mask_j + pair_ij:
//
//     p_ij    = exp(t_ij - LSE_i)
//     delta_i = dO_i . O_i                    (= sum_j p_ij dO_i . v_j)
//     dt_ij   = p_ij (dO_i . v_j - delta_i)
//     dQ_i = sum_j dt_ij k_j / sqrt(D),  dK_j = sum_i dt_ij q_i / sqrt(D),
//     dV_j = sum_i p_ij dO_i,
//     dmask[b,n,j] = sum_h sum_i dt_ij,  dpair[b,h,i,j] = sum_n dt_ij.
//
// Mask rebase.  As in the forward kernels, the mask of each (b, n) is shifted
// by its maximum c (a constant shift of every logit of the row, which changes
// no weight), so logits and LSE_i - c stay small numbers.  The forward's LSE
// is an fp32 number; where |c| is large (a row whose every key carries the
// guide's -1e9) its fp32 rounding (64 at 1e9) would swamp LSE_i - c, so the
// row statistics recompute log sum_j exp(t_ij - c) for those rows
// from Q, K and the biases instead of subtracting.
#pragma once

#include <cstdint>

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "fwd_f32.cuh"

namespace evo {

// |c| above which the row statistics are recomputed rather than taken from
// the forward's LSE (fp32 spacing at 4096 is 2^-11, so LSE - c keeps an
// error below 2.5e-4 up to here).
constexpr float kBwdRecomputeAbove = 4096.f;
constexpr int kBwdChunk = 32;  // output columns (of D) per SIMT thread

template <typename T>  // float, uint16_t holding bf16, or __half
struct BwdParams {
    const T* q;
    const T* k;
    const T* v;
    const T* mask;   // [B, N, S] or nullptr
    const T* pair;   // [B, H, S, S] or nullptr
    const T* o;
    const T* dout;
    const float* lse;  // [B, N, H, S], from the forward
    T* dq;
    T* dk;
    T* dv;
    T* dmask;  // [B, N, S] or nullptr (not requested)
    T* dpair;  // [B, H, S, S] or nullptr (not requested)
    float* cmask;   // workspace [B * N]: the mask rebase c of each (b, n)
    float* lse_r;   // workspace [B, N, H, S]: LSE - c (natural log); +inf for rows without a finite logit
    float* delta;   // workspace [B, N, H, S]: dO . O
    int* shifted;   // workspace [1 + B * N]: count, then the (b, n) whose rows need the LSE recomputed
    int B, N, S, H, D;
    int vec16;      // 16-bit elements, D % 8 == 0 and O, dO, K 16-byte aligned: rows read 16 bytes at a time
    float scale;    // 1 / sqrt(D)
};

// The mask rebase c of each (b, n): one warp per (b, n).
template <typename T>
__global__ void __launch_bounds__(256) evo_bwd_shift_kernel(const BwdParams<T> p, long long bns) {
    const long long bn = blockIdx.x * 8ll + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (bn >= bns) return;
    float c = 0.f;
    if (p.mask != nullptr) {
        const T* mrow = p.mask + size_t(bn) * p.S;
        float mx = -INFINITY;
        for (int j = lane; j < p.S; j += 32) mx = fmaxf(mx, ld_elem(mrow, j));
        mx = warp_max(mx);
        c = (mx == -INFINITY) ? 0.f : mx;
    }
    if (lane == 0) {
        p.cmask[bn] = c;
        if (fabsf(c) > kBwdRecomputeAbove) p.shifted[1 + atomicAdd(p.shifted, 1)] = int(bn);
    }
}

// delta and LSE - c of every row: one thread per (b, n, i, h) row, in memory
// order (the thread's O and dO rows are D consecutive elements).  Rows of an
// n whose shift |c| exceeds kBwdRecomputeAbove get their LSE - c from
// evo_bwd_lse_recompute_kernel instead.
template <typename T>
__global__ void __launch_bounds__(256) evo_bwd_rowstats_kernel(const BwdParams<T> p, long long rows) {
    const long long r = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    if (r >= rows) return;
    const int D = p.D;
    const int h = int(r % p.H);
    const long long bi = r / p.H;  // bn * S + i
    const int i = int(bi % p.S);
    const long long bn = bi / p.S;
    const size_t off = size_t(r) * D;
    float acc = 0.f;
    bool done = false;
    if constexpr (sizeof(T) == 2) {
        if (p.vec16) {
            // 8 elements per 16-byte load
            const uint4* o4 = reinterpret_cast<const uint4*>(p.o + off);
            const uint4* g4 = reinterpret_cast<const uint4*>(p.dout + off);
            for (int d = 0; d < D / 8; ++d) {
                const uint4 a = o4[d], g = g4[d];
                const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, gw[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const T* ae = reinterpret_cast<const T*>(&aw[e]);
                    const T* ge = reinterpret_cast<const T*>(&gw[e]);
                    acc = fmaf(ld_elem(ae, 0), ld_elem(ge, 0), acc);
                    acc = fmaf(ld_elem(ae, 1), ld_elem(ge, 1), acc);
                }
            }
            done = true;
        }
    }
    if (!done)
        for (int d = 0; d < D; ++d) acc = fmaf(ld_elem(p.o, off + d), ld_elem(p.dout, off + d), acc);
    const size_t ri = (size_t(bn) * p.H + h) * p.S + i;
    p.delta[ri] = acc;
    const float c = p.cmask[bn];
    if (!(fabsf(c) > kBwdRecomputeAbove)) {
        const float L = p.lse[ri];
        p.lse_r[ri] = (L == -INFINITY) ? INFINITY : L - c;
    }
}

// LSE - c recomputed from the inputs, log sum_j exp(t_ij - c), for the rows
// of every n whose shift |c| exceeds kBwdRecomputeAbove (the forward's fp32
// LSE near such a c has lost the digits that matter).  Those n are listed by
// evo_bwd_shift_kernel; a grid of a few blocks per SM walks their rows, one
// warp per row, lanes over keys, the query row staged in shared memory.
template <typename T>
__global__ void __launch_bounds__(256) evo_bwd_lse_recompute_kernel(const BwdParams<T> p) {
    __shared__ float qs[8][kF32MaxD];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long rows_per_n = (long long)p.H * p.S;
    const long long total = (long long)p.shifted[0] * rows_per_n;
    const long long nwarps = (long long)gridDim.x * 8;
    const int D = p.D;
    const size_t row_stride = size_t(p.H) * D;
    for (long long w = blockIdx.x * 8ll + warp; w < total; w += nwarps) {
        const long long bn = p.shifted[1 + w / rows_per_n];
        const int r = int(w % rows_per_n);
        const int h = r / p.S, i = r - h * p.S;
        const long long b = bn / p.N;
        const float c = p.cmask[bn];
        const T* mrow = p.mask + size_t(bn) * p.S;
        const size_t qoff = (size_t(bn) * p.S + i) * row_stride + size_t(h) * D;
        for (int d = lane; d < D; d += 32) qs[warp][d] = ld_elem(p.q, qoff + d);
        __syncwarp();
        const T* prow = p.pair ? p.pair + ((size_t(b) * p.H + h) * p.S + i) * size_t(p.S) : nullptr;
        float m = -INFINITY, s = 0.f;
        for (int j = lane; j < p.S; j += 32) {
            const size_t koff = (size_t(bn) * p.S + j) * row_stride + size_t(h) * D;
            float dot = 0.f;
            bool done = false;
            if constexpr (sizeof(T) == 2) {
                if (p.vec16) {
                    const uint4* k4 = reinterpret_cast<const uint4*>(p.k + koff);
                    for (int d8 = 0; d8 < D / 8; ++d8) {
                        const uint4 kv = __ldg(k4 + d8);
                        const uint32_t kw[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const T* ke = reinterpret_cast<const T*>(&kw[e]);
                            dot = fmaf(qs[warp][8 * d8 + 2 * e], ld_elem(ke, 0), dot);
                            dot = fmaf(qs[warp][8 * d8 + 2 * e + 1], ld_elem(ke, 1), dot);
                        }
                    }
                    done = true;
                }
            }
            if (!done)
                for (int d = 0; d < D; ++d) dot = fmaf(qs[warp][d], ld_elem(p.k, koff + d), dot);
            float t = dot * p.scale + (ld_elem(mrow, j) - c);
            if (prow) t += ld_elem(prow, j);
            if (t > m) {
                s = s * expf(m - t) + 1.f;  // m = -inf gives s * 0 + 1
                m = t;
            } else if (t > -INFINITY) {
                s += expf(t - m);
            }
        }
        const float mw = warp_max(m);
        const float sw = warp_sum(m == -INFINITY ? 0.f : s * expf(m - mw));
        if (lane == 0) p.lse_r[(size_t(bn) * p.H + h) * p.S + i] = (mw == -INFINITY) ? INFINITY : mw + logf(sw);
        __syncwarp();
    }
}

// The weight p_ij and logit gradient dt_ij of one (query i, key j) pair of
// slice (bn, h), recomputed from the inputs (all loads through L1).
template <typename T>
__device__ __forceinline__ void bwd_pair_terms(const BwdParams<T>& p, long long bn, long long b, int h, int i, int j,
                                               float c, float* pij, float* dtij) {
    const size_t row_stride = size_t(p.H) * p.D;
    const size_t qoff = (size_t(bn) * p.S + i) * row_stride + size_t(h) * p.D;
    const size_t koff = (size_t(bn) * p.S + j) * row_stride + size_t(h) * p.D;
    const size_t ri = (size_t(bn) * p.H + h) * p.S + i;
    const float lr = p.lse_r[ri];
    if (lr == INFINITY) {
        *pij = 0.f;
        *dtij = 0.f;
        return;
    }
    float dot = 0.f, dp = 0.f;
    for (int d = 0; d < p.D; ++d) {
        dot = fmaf(ld_elem(p.q, qoff + d), ld_elem(p.k, koff + d), dot);
        dp = fmaf(ld_elem(p.dout, qoff + d), ld_elem(p.v, koff + d), dp);
    }
    float t = dot * p.scale;
    if (p.mask) t += ld_elem(p.mask, size_t(bn) * p.S + j) - c;
    if (p.pair) t += ld_elem(p.pair, ((size_t(b) * p.H + h) * p.S + i) * size_t(p.S) + j);
    const float pw = expf(t - lr);
    *pij = pw;
    *dtij = pw * (dp - p.delta[ri]);
}

// dK and dV: one thread per (b, n, h, key j, chunk of 32 columns).
template <typename T>
__global__ void __launch_bounds__(128) evo_bwd_simt_kv_kernel(const BwdParams<T> p, long long total) {
    const long long t = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    if (t >= total) return;
    const int nch = (p.D + kBwdChunk - 1) / kBwdChunk;
    const int ch = int(t % nch);
    long long r = t / nch;
    const int j = int(r % p.S);
    r /= p.S;
    const int h = int(r % p.H);
    const long long bn = r / p.H;
    const long long b = bn / p.N;
    const float c = p.cmask[bn];
    const int d0 = ch * kBwdChunk;
    const int nd = min(kBwdChunk, p.D - d0);
    float ak[kBwdChunk], av[kBwdChunk];
#pragma unroll
    for (int e = 0; e < kBwdChunk; ++e) ak[e] = av[e] = 0.f;
    const size_t row_stride = size_t(p.H) * p.D;
    for (int i = 0; i < p.S; ++i) {
        float pw, dt;
        bwd_pair_terms(p, bn, b, h, i, j, c, &pw, &dt);
        if (pw == 0.f && dt == 0.f) continue;
        const size_t qoff = (size_t(bn) * p.S + i) * row_stride + size_t(h) * p.D + d0;
#pragma unroll
        for (int e = 0; e < kBwdChunk; ++e)
            if (e < nd) {
                ak[e] = fmaf(dt, ld_elem(p.q, qoff + e), ak[e]);
                av[e] = fmaf(pw, ld_elem(p.dout, qoff + e), av[e]);
            }
    }
    const size_t koff = (size_t(bn) * p.S + j) * row_stride + size_t(h) * p.D + d0;
#pragma unroll
    for (int e = 0; e < kBwdChunk; ++e)
        if (e < nd) {
            st_elem(p.dk, koff + e, ak[e] * p.scale);
            st_elem(p.dv, koff + e, av[e]);
        }
}

// dQ: one thread per (b, n, h, query i, chunk of 32 columns).
template <typename T>
__global__ void __launch_bounds__(128) evo_bwd_simt_q_kernel(const BwdParams<T> p, long long total) {
    const long long t = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    if (t >= total) return;
    const int nch = (p.D + kBwdChunk - 1) / kBwdChunk;
    const int ch = int(t % nch);
    long long r = t / nch;
    const int i = int(r % p.S);
    r /= p.S;
    const int h = int(r % p.H);
    const long long bn = r / p.H;
    const long long b = bn / p.N;
    const float c = p.cmask[bn];
    const int d0 = ch * kBwdChunk;
    const int nd = min(kBwdChunk, p.D - d0);
    float aq[kBwdChunk];
#pragma unroll
    for (int e = 0; e < kBwdChunk; ++e) aq[e] = 0.f;
    const size_t row_stride = size_t(p.H) * p.D;
    for (int j = 0; j < p.S; ++j) {
        float pw, dt;
        bwd_pair_terms(p, bn, b, h, i, j, c, &pw, &dt);
        if (dt == 0.f) continue;
        const size_t koff = (size_t(bn) * p.S + j) * row_stride + size_t(h) * p.D + d0;
#pragma unroll
        for (int e = 0; e < kBwdChunk; ++e)
            if (e < nd) aq[e] = fmaf(dt, ld_elem(p.k, koff + e), aq[e]);
    }
    const size_t qoff = (size_t(bn) * p.S + i) * row_stride + size_t(h) * p.D + d0;
#pragma unroll
    for (int e = 0; e < kBwdChunk; ++e)
        if (e < nd) st_elem(p.dq, qoff + e, aq[e] * p.scale);
}

// dmask: one thread per (b, n, key j), summing dt over heads and query rows.
template <typename T>
__global__ void __launch_bounds__(128) evo_bwd_simt_dmask_kernel(const BwdParams<T> p, long long total) {
    const long long t = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    if (t >= total) return;
    const int j = int(t % p.S);
    const long long bn = t / p.S;
    const long long b = bn / p.N;
    const float c = p.cmask[bn];
    float acc = 0.f;
    for (int h = 0; h < p.H; ++h)
        for (int i = 0; i < p.S; ++i) {
            float pw, dt;
            bwd_pair_terms(p, bn, b, h, i, j, c, &pw, &dt);
            acc += dt;
        }
    st_elem(p.dmask, size_t(bn) * p.S + j, acc);
}

// dpair: one thread per (b, h, query i, key j), summing dt over n.
template <typename T>
__global__ void __launch_bounds__(128) evo_bwd_simt_dpair_kernel(const BwdParams<T> p, long long total) {
    const long long t = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    if (t >= total) return;
    const int j = int(t % p.S);
    long long r = t / p.S;
    const int i = int(r % p.S);
    r /= p.S;
    const int h = int(r % p.H);
    const long long b = r / p.H;
    float acc = 0.f;
    for (int n = 0; n < p.N; ++n) {
        const long long bn = b * p.N + n;
        float pw, dt;
        bwd_pair_terms(p, bn, b, h, i, j, p.cmask[bn], &pw, &dt);
        acc += dt;
    }
    st_elem(p.dpair, size_t(t), acc);
}

}  // namespace evo
