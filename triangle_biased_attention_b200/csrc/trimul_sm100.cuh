// Triangle multiplication on sm_100a: the contraction over the third node of
// two edge representations, channel by channel (bf16 / fp16 in, fp32
// accumulation, output in the input type).
//
// The NVIDIA cuEquivariance blog (open-lab.net, "Accelerated molecular
// modeling with NVIDIA cuEquivariance and NVIDIA NIM microservices", the
// triangle-operations sections) names triangle multiplication beside triangle
// attention as the O(N^3) operations of these models ("triangular
// relationships": i close to k and k close to j relate i and j).  It prints no
// formula; the reading implemented here, per batch entry b and channel c:
//
//     outgoing:  Z[i, j] = sum_k A[i, k] B[j, k]      (Z_c = A_c B_c^T)
//     incoming:  Z[i, j] = sum_k A[k, i] B[k, j]      (Z_c = A_c^T B_c)
//
// with A, B, Z laid out [Bt, N, N, C] (channels last).  Three kernels:
//  * a tiled transpose to channel-first [Bt*C, N, Np] (Np = N rounded up to
//    8, so that every row is a whole number of 16-byte units for TMA);
//  * a persistent tcgen05 batched GEMM over the (b, c) channel matrices,
//    128 x 256 output tiles, K in steps of 64 through a 4-stage TMA ring, the
//    fp32 accumulator double-buffered in tensor memory so that a tile's
//    epilogue overlaps the next tile's MMAs.  Outgoing reads both operands
//    K-major (k contiguous: rows of the channel-first copies); incoming reads
//    both MN-major (i or j contiguous), the same copies read the other way;
//  * the transpose back to [Bt, N, N, C].
// Every wait is bounded (2 s); on expiry the CTA records EVO_ERR_TIMEOUT,
// drains its own copies and MMAs, frees tensor memory and exits.
#pragma once

#include <cuda.h>
#include <cstdint>

#include "common.cuh"
#include "ptx_sm100.cuh"
#include "tile_sm100.cuh"

namespace evo {

// ------------------------------------------------------------------ transposes

// X[b, p, q, c] (q < N, channels last) -> Y[(b * C + c), p, q] with row
// stride ldq (>= N).  One block per (b, p) (grid x) and 32 x 32 tile of
// (q, c) (grid y, z).
template <typename T>
__global__ void __launch_bounds__(256) evo_trimul_to_cfirst(const T* __restrict__ x, T* __restrict__ y, int N,
                                                            int C, int ldq) {
    __shared__ T tile[32][33];
    const int q0 = blockIdx.y * 32, c0 = blockIdx.z * 32;
    const long long bp = blockIdx.x;  // b * N + p
    const long long b = bp / N;
    const int p = int(bp - b * N);
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8
    for (int r = ty; r < 32; r += 8) {
        const int q = q0 + r, c = c0 + tx;
        if (q < N && c < C) tile[r][tx] = x[(size_t(bp) * N + q) * C + c];
    }
    __syncthreads();
    for (int r = ty; r < 32; r += 8) {
        const int c = c0 + r, q = q0 + tx;
        if (q < N && c < C) y[((size_t(b) * C + c) * N + p) * size_t(ldq) + q] = tile[tx][r];
    }
}

// Y[(b * C + c), i, j] (row stride ldj) -> Z[b, i, j, c].  One block per
// (b, i) (grid x) and 32 x 32 tile of (j, c) (grid y, z).
template <typename T>
__global__ void __launch_bounds__(256) evo_trimul_to_clast(const T* __restrict__ y, T* __restrict__ z, int N, int C,
                                                           int ldj) {
    __shared__ T tile[32][33];
    const int j0 = blockIdx.y * 32, c0 = blockIdx.z * 32;
    const long long bi = blockIdx.x;  // b * N + i
    const long long b = bi / N;
    const int i = int(bi - b * N);
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
    for (int r = ty; r < 32; r += 8) {
        const int c = c0 + r, j = j0 + tx;
        if (j < N && c < C) tile[r][tx] = y[((size_t(b) * C + c) * N + i) * size_t(ldj) + j];
    }
    __syncthreads();
    for (int r = ty; r < 32; r += 8) {
        const int j = j0 + r, c = c0 + tx;
        if (j < N && c < C) z[(size_t(bi) * N + j) * C + c] = tile[tx][r];
    }
}

// The same two transposes with 16-byte global accesses, for C a multiple of 8
// and 16-byte aligned pointers: a block moves a 64 x 64 tile (rows of 8
// 16-byte vectors on both sides) through shared memory; 256 threads, 2
// vectors each.
// Writes of the channel-first copies may run into the row padding (columns
// N .. ldq - 1), which is never read.
// Element (row, col) of a 64 x 64 16-bit tile in shared memory: rows of 128 B,
// the 16-byte vector index XORed with bits 3-5 of the row, so that a column
// read by 8 threads 8 rows apart falls in 8 different banks.
__device__ __forceinline__ int tr_idx(int row, int col) {
    return row * 64 + ((((col >> 3) ^ (row >> 3)) & 7) << 3) + (col & 7);
}

template <typename T>
__global__ void __launch_bounds__(256) evo_trimul_to_cfirst_v(const T* __restrict__ x, T* __restrict__ y, int N,
                                                              int C, int ldq) {
    __shared__ __align__(16) uint16_t tile[64 * 64];  // [q][c]
    const int q0 = blockIdx.y * 64, c0 = blockIdx.z * 64;
    const long long bp = blockIdx.x;
    const long long b = bp / N;
    const int p = int(bp - b * N);
    const uint16_t* xs = reinterpret_cast<const uint16_t*>(x);
    uint16_t* ys = reinterpret_cast<uint16_t*>(y);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int v = threadIdx.x + 256 * h;  // 64 rows (q) x 8 vectors (c)
        const int r = v >> 3, cv = (v & 7) * 8;
        const int q = q0 + r, c = c0 + cv;
        uint4 val = make_uint4(0u, 0u, 0u, 0u);
        if (q < N && c < C) val = *reinterpret_cast<const uint4*>(xs + (size_t(bp) * N + q) * C + c);
        *reinterpret_cast<uint4*>(&tile[tr_idx(r, cv)]) = val;
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int v = threadIdx.x + 256 * h;  // 64 rows (c) x 8 vectors (q)
        const int r = v >> 3, qv = (v & 7) * 8;
        const int c = c0 + r, q = q0 + qv;
        if (c < C && q < ldq) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
                w[e] = uint32_t(tile[tr_idx(qv + 2 * e, r)]) | (uint32_t(tile[tr_idx(qv + 2 * e + 1, r)]) << 16);
            *reinterpret_cast<uint4*>(ys + ((size_t(b) * C + c) * N + p) * size_t(ldq) + q) =
                make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
}

template <typename T>
__global__ void __launch_bounds__(256) evo_trimul_to_clast_v(const T* __restrict__ y, T* __restrict__ z, int N,
                                                             int C, int ldj) {
    __shared__ __align__(16) uint16_t tile[64 * 64];  // [c][j]
    const int j0 = blockIdx.y * 64, c0 = blockIdx.z * 64;
    const long long bi = blockIdx.x;
    const long long b = bi / N;
    const int i = int(bi - b * N);
    const uint16_t* ys = reinterpret_cast<const uint16_t*>(y);
    uint16_t* zs = reinterpret_cast<uint16_t*>(z);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int v = threadIdx.x + 256 * h;  // 64 rows (c) x 8 vectors (j)
        const int r = v >> 3, jv = (v & 7) * 8;
        const int c = c0 + r, j = j0 + jv;
        uint4 val = make_uint4(0u, 0u, 0u, 0u);
        if (c < C && j < ldj)
            val = *reinterpret_cast<const uint4*>(ys + ((size_t(b) * C + c) * N + i) * size_t(ldj) + j);
        *reinterpret_cast<uint4*>(&tile[tr_idx(r, jv)]) = val;
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int v = threadIdx.x + 256 * h;  // 64 rows (j) x 8 vectors (c)
        const int r = v >> 3, cv = (v & 7) * 8;
        const int j = j0 + r, c = c0 + cv;
        if (j < N && c < C) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
                w[e] = uint32_t(tile[tr_idx(cv + 2 * e, r)]) | (uint32_t(tile[tr_idx(cv + 2 * e + 1, r)]) << 16);
            *reinterpret_cast<uint4*>(zs + (size_t(bi) * N + j) * C + c) = make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
}

// --------------------------------------------------------------- batched GEMM

struct TrimulParams {
    uint16_t* zc;    // [Bt*C, N, ldz] channel-first result (bf16 / fp16 bits)
    int N, ldz;
    int tiles_m;     // ceil(N / 128): row blocks
    int tiles_n;     // ceil(N / BN): column blocks
    int num_tiles;   // Bt * C * tiles_m * tiles_n
    int k_steps;     // ceil(N / 64)
};

// Output tiles of 128 rows x BN = 256 columns: one M = 128, N = 256 MMA per
// 16-deep K step (an MMA instruction costs about the same time at N = 256 as
// at N = 128, so the wider tile halves the instructions per flop).
template <bool OUTGOING, bool F16>
struct TrimulCfg {
    static constexpr int THREADS = 256;  // warp 0 loads, warp 1 MMAs, warps 4-7 epilogue
    static constexpr int BN = 256;
    static constexpr int STAGES = 4;
    static constexpr int OPER = 128 * 128;             // A stage: 128 rows x 64 k of bf16 = 16 KB
    static constexpr int OPER_B = BN * 128;            // B stage: BN x 64 k = 32 KB
    static constexpr int STAGE_BYTES = OPER + OPER_B;
    static constexpr int OFF_BAR = STAGES * STAGE_BYTES;
    static constexpr int BAR_FULL = 0, BAR_EMPTY = STAGES, BAR_AF = 2 * STAGES, BAR_AE = 2 * STAGES + 2,
                         BAR_DRAIN = 2 * STAGES + 4, NUM_BARS = 2 * STAGES + 5;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
    static constexpr uint32_t TMEM_COLS = 2 * BN;      // two BN-column accumulators
    static constexpr uint32_t AB = F16 ? 0u : ((1u << 7) | (1u << 10));
    static constexpr uint32_t MAJ = OUTGOING ? 0u : ((1u << 15) | (1u << 16));
    static constexpr uint32_t IDESC =
        (1u << 4) | AB | MAJ | ((uint32_t(BN) >> 3) << 17) | ((128u >> 4) << 24);
};

template <bool OUTGOING, bool F16>
__global__ void __launch_bounds__(256, 1)
evo_trimul_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                       const TrimulParams p) {
    using C = TrimulCfg<OUTGOING, F16>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = ptx::smem_u32(smem);
    const int warp = __shfl_sync(0xffffffffu, int(threadIdx.x >> 5), 0);
    const int lane = threadIdx.x & 31;
    const int G = gridDim.x;
    auto bar = [&](int i) -> uint32_t { return sb + C::OFF_BAR + 8u * uint32_t(i); };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
    // tile L: column block fastest, then row block, then channel matrix
    auto tile = [&](int L, int& tj, int& ti, int& bc) {
        tj = L % p.tiles_n;
        const int r = L / p.tiles_n;
        ti = r % p.tiles_m;
        bc = r / p.tiles_m;
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            ptx::mbar_init(bar(C::BAR_FULL + s), 1);
            ptx::mbar_init(bar(C::BAR_EMPTY + s), 1);
        }
        for (int a = 0; a < 2; ++a) {
            ptx::mbar_init(bar(C::BAR_AF + a), 1);
            ptx::mbar_init(bar(C::BAR_AE + a), 4);
        }
        ptx::mbar_init(bar(C::BAR_DRAIN), 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc(ptx::smem_u32(tmem_slot), C::TMEM_COLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // -------------------------------------------------------------- loads
        if (lane == 0) {
            ptx::prefetch_tmap(&tm_a);
            ptx::prefetch_tmap(&tm_b);
        }
        int n = 0;
        bool ok = true;
        for (int L = blockIdx.x; L < p.num_tiles && ok; L += G) {
            int tj, ti, bc;
            tile(L, tj, ti, bc);
            for (int kt = 0; kt < p.k_steps; ++kt, ++n) {
                const int s = n % C::STAGES;
                ok = wait_warp(bar(C::BAR_EMPTY + s), ((n / C::STAGES) & 1) ^ 1, abort_flag);
                if (!ok) break;
                if (lane == 0) {
                    const uint32_t a = sb + uint32_t(s * C::STAGE_BYTES), b = a + C::OPER;
                    const uint32_t f = bar(C::BAR_FULL + s);
                    ptx::mbar_arrive_expect_tx(f, C::STAGE_BYTES);
                    // 64 x 64 boxes: outgoing, rows i (resp. j) of 64 k each; incoming,
                    // rows k of 64 i (resp. j) each
#pragma unroll
                    for (int x = 0; x < 2; ++x) {
                        if (OUTGOING) ptx::tma_load_3d(a + 8192 * x, &tm_a, f, 64 * kt, 128 * ti + 64 * x, bc);
                        else ptx::tma_load_3d(a + 8192 * x, &tm_a, f, 128 * ti + 64 * x, 64 * kt, bc);
                    }
#pragma unroll
                    for (int x = 0; x < C::BN / 64; ++x) {
                        if (OUTGOING) ptx::tma_load_3d(b + 8192 * x, &tm_b, f, 64 * kt, C::BN * tj + 64 * x, bc);
                        else ptx::tma_load_3d(b + 8192 * x, &tm_b, f, C::BN * tj + 64 * x, 64 * kt, bc);
                    }
                }
                __syncwarp();
            }
        }
        if (!ok && lane == 0) {
            // the last load of each stage lands before the CTA exits
            for (int s = 0; s < C::STAGES; ++s)
                if (n - 1 >= s) {
                    const int last = s + C::STAGES * ((n - 1 - s) / C::STAGES);
                    wait_bounded(bar(C::BAR_FULL + s), uint32_t(last / C::STAGES) & 1u, nullptr);
                }
        }
        __syncwarp();
    } else if (warp == 1) {
        // --------------------------------------------------------------- MMAs
        int n = 0, t = 0;
        bool ok = true, issued = false;
        for (int L = blockIdx.x; L < p.num_tiles && ok; L += G, ++t) {
            const int acc = t & 1;
            // the epilogue has drained this accumulator's previous tile
            ok = wait_warp(bar(C::BAR_AE + acc), ((t >> 1) & 1) ^ 1, abort_flag);
            if (!ok) break;
            ptx::tc_fence_after();
            const uint32_t d = tmem + uint32_t(C::BN * acc);
            for (int kt = 0; kt < p.k_steps; ++kt, ++n) {
                const int s = n % C::STAGES;
                ok = wait_warp(bar(C::BAR_FULL + s), uint32_t(n / C::STAGES) & 1u, abort_flag);
                if (!ok) break;
                ptx::tc_fence_after();
                const uint32_t a = sb + uint32_t(s * C::STAGE_BYTES), b = a + C::OPER;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    uint64_t da, db;
                    if (OUTGOING) {
                        // K-major: 128 rows of 128 B; K step kk is 32 B into each row
                        da = desc_k_major<128>(a + 32 * kk);
                        db = desc_k_major<128>(b + 32 * kk);
                    } else {
                        // MN-major: rows are k (128 B of i or j each), 64-wide atoms 8 KB apart
                        da = desc_mn_major<128>(a + 2048 * kk, 8192);
                        db = desc_mn_major<128>(b + 2048 * kk, 8192);
                    }
                    ptx::mma_ss_elect(d, da, db, C::IDESC, (kt > 0 || kk > 0) ? 1u : 0u);
                }
                issued = true;
                ptx::mma_commit_elect(bar(C::BAR_EMPTY + s));
            }
            if (!ok) break;
            ptx::mma_commit_elect(bar(C::BAR_AF + acc));
        }
        if (!ok && issued) {
            ptx::mma_commit_elect(bar(C::BAR_DRAIN));
            wait_bounded(bar(C::BAR_DRAIN), 0, nullptr);
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ----------------------------------------------------------- epilogue
        const int wq = warp - 4;
        const int r = 32 * wq + lane;
        const uint32_t tl = tmem + (uint32_t(32 * wq) << 16);
        int t = 0;
        bool ok = true;
        for (int L = blockIdx.x; L < p.num_tiles && ok; L += G, ++t) {
            int tj, ti, bc;
            tile(L, tj, ti, bc);
            const int acc = t & 1;
            ok = wait_warp(bar(C::BAR_AF + acc), uint32_t(t >> 1) & 1u, abort_flag);
            if (!ok) break;
            ptx::tc_fence_after();
            const int i = 128 * ti + r;
            uint16_t* row = p.zc + (size_t(bc) * p.N + i) * size_t(p.ldz);
#pragma unroll 1
            for (int c4 = 0; c4 < C::BN / 32; ++c4) {
                float v[32];
                ptx::tmem_ld_x32(tl + uint32_t(C::BN * acc + 32 * c4), reinterpret_cast<uint32_t*>(v));
                ptx::tmem_ld_wait_x32(reinterpret_cast<uint32_t*>(v));
                if (c4 == C::BN / 32 - 1) {
                    ptx::tc_fence_before();
                    ptx::mbar_arrive_elect(bar(C::BAR_AE + acc));
                }
                if (i < p.N) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int j = C::BN * tj + 32 * c4 + 8 * e;
                        if (j < p.ldz) {
                            uint4 o;
                            if constexpr (F16) {
                                o = make_uint4(ptx::pack_f16x2(v[8 * e], v[8 * e + 1]),
                                               ptx::pack_f16x2(v[8 * e + 2], v[8 * e + 3]),
                                               ptx::pack_f16x2(v[8 * e + 4], v[8 * e + 5]),
                                               ptx::pack_f16x2(v[8 * e + 6], v[8 * e + 7]));
                            } else {
                                o = make_uint4(ptx::pack_bf16x2(v[8 * e], v[8 * e + 1]),
                                               ptx::pack_bf16x2(v[8 * e + 2], v[8 * e + 3]),
                                               ptx::pack_bf16x2(v[8 * e + 4], v[8 * e + 5]),
                                               ptx::pack_bf16x2(v[8 * e + 6], v[8 * e + 7]));
                            }
                            *reinterpret_cast<uint4*>(row + j) = o;
                        }
                    }
                }
            }
        }
        (void)ok;
    }

    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == 1) ptx::tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace evo
