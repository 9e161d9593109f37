// Biased-attention backward on sm_100a (bf16 / fp16, head dims 16, 32, 64):
// one CTA per SM walking (b, n, h, 128-key block) units, tcgen05 MMAs with
// fp32 accumulators in tensor memory.
//
// What it computes is the chain rule of the forward formula, as the backward
// kernel of the DeepSpeed DS4Sci_EvoformerAttention guide (hmyw.cn, sections
// 1 and 5.4) is described: the attention weights are recomputed from Q, K and
// the forward's log-sum-exp (never stored), delta = dO . O is a per-row
// intermediate, and the bias gradients are computed only when asked for.  Per
// unit (one key block of one slice) and query block:
//
//     S  = Q K^T            (MMA, M = 128 queries, N = 128 keys, K = D)
//     dP = dO V^T           (MMA, same shape)
//     P  = 2^(S log2(e)/sqrt(D) + (mask - c + pair) log2(e) - (LSE - c) log2(e))
//     dT = P (dP - delta)   (the logit gradient; softmax warps, one query row
//                            per thread, written to shared memory as bf16/fp16)
//     dV     += P^T dO      (MMA, M = 128 keys, K = 128 queries, N = D)
//     dK_aug += dT^T [Q | 1] (N = D + 16: column D is the column sum of dT,
//                            this head's share of dmask for the block's keys)
//     dQ      = dT K        (MMA, M = 128 queries, N = D), added to an fp32
//                            accumulator in global memory (every key block of
//                            the slice contributes)
//     dpair  += dT          (fp32, into global memory: the pair bias is shared
//                            by every n)
//
// Both global sums are TMA tile reductions (cp.reduce.async.bulk.tensor
// .add): a warp stages its 32 rows in shared memory and one lane issues the
// reduction, so L2 adds whole 128 B (dpair) or 64 B (dQ) rows instead of the
// 16 B pieces of per-thread vector atomics.
//
// dK and dV stay in tensor memory for the whole unit and are written once; the
// fp32 dQ, dmask and dpair sums are rounded to the output type by a final
// kernel.  Layouts: every Q, K, V, dO tile is loaded by TMA as D/16 boxes of
// 128 rows x 16 columns (32 B rows, 32 B swizzle), so the same bytes serve as
// a K-major operand (S, dP) and as an MN-major one (dV, dK, dQ); the Q stage
// carries one more box holding 1 in its first column (the ones column of
// dK_aug).  P and dT tiles are two 64-key atoms of 128 B rows (128 B
// swizzle): K-major for dQ (keys along K), MN-major for dV and dK (keys along
// M).  Warp roles: warp 0 loads, warp 1 issues the MMAs (one elected lane of
// the converged warp); one (D = 64) or two (D <= 32) softmax warpgroups
// compute P and dT (a thread owns one query row; with two groups, each takes
// 64 of its 128 keys, so the step's P and dT are written in half the time);
// the last warpgroup drains dQ, dK, dV and the dmask column out of tensor
// memory.  Every wait is bounded; on expiry the CTA records
// EVO_ERR_TIMEOUT, lets its own copies and MMAs finish, frees tensor memory and
// exits.
#pragma once

#include <cuda.h>
#include <cstdint>

#include "common.cuh"
#include "ptx_sm100.cuh"
#include "tile_sm100.cuh"

namespace evo {

struct BwdTriParams {
    const uint16_t* mask;  // [B, N, S] bf16/fp16 bits, or nullptr
    const float* cmask;    // [B * N] mask rebase c
    const float* lse_r;    // [B, N, H, S] LSE - c (natural log); +inf: no finite logit
    const float* delta;    // [B, N, H, S] dO . O
    uint16_t* dk;          // [B, N, S, H, D]
    uint16_t* dv;          // [B, N, S, H, D]
    float* dq_acc;         // [B, N, S, H, D] fp32, zero on entry
    float* dmask_acc;      // [B, N, S] fp32, zero on entry, or nullptr (not requested)
    float* dpair_acc;      // [B, H, S, S] fp32, zero on entry, or nullptr (not requested)
    int N, S, H;
    int num_kb, num_qb;
    int num_units;         // B * N * H * num_kb
    float scale_log2;      // log2(e) / sqrt(D)
    float scale;           // 1 / sqrt(D)
};

template <int D, bool HAS_PAIR, bool F16>
struct BwdCfg {
    static_assert(D == 16 || D == 32 || D == 64, "head dim");
    // softmax warpgroups: 2 at D <= 32, each taking 64 of a row's 128 keys (so
    // that a step's P and dT are written twice as fast), 1 at D = 64 (whose
    // epilogue needs more registers than the split leaves)
    static constexpr int GROUPS = D <= 32 ? 2 : 1;
    static constexpr int THREADS = 128 * (2 + GROUPS);
    static constexpr int EPI0 = 4 + 4 * GROUPS;  // first epilogue warp
    static constexpr int LOW_REGS = 80, HIGH_REGS = 144;  // setmaxnreg split at GROUPS = 2
    static_assert(GROUPS == 1 || 128 * LOW_REGS + 3 * 128 * HIGH_REGS <= 65536, "register split");
    static constexpr int BOX = kBM * 32;         // 128 rows x 16 columns, 32 B swizzle
    static constexpr int NBOX = D / 16;
    static constexpr int TILE = NBOX * BOX;      // one Q, K, V or dO tile
    static constexpr int QAUG = TILE + BOX;      // Q tile + the ones box
    static constexpr int KV_STAGES = D <= 32 ? 2 : 1;
    static constexpr int Q_STAGES = 2;
    // pair-bias tiles as a ring of half tiles (128 query rows x 64 keys, 128 B
    // swizzle): a step uses two, halves 2g and 2g + 1, each read by the
    // softmax warps of its keys
    static constexpr int PAIR_SLOTS = HAS_PAIR ? (GROUPS == 2 ? 3 : (D <= 32 ? 4 : 2)) : 0;
    static constexpr int PAIR_RING = HAS_PAIR ? PAIR_SLOTS : 1;
    static constexpr int HALF_BYTES = kBM * 64 * 2;
    static constexpr int PT_ATOM = kBM * 128;          // 64 keys x 128 rows
    static constexpr int PT_BYTES = 2 * PT_ATOM;       // P or dT tile
    // shared-memory map (every tile 1024-aligned)
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = OFF_K + KV_STAGES * TILE;
    static constexpr int OFF_Q = OFF_V + KV_STAGES * TILE;
    static constexpr int OFF_DO = OFF_Q + Q_STAGES * QAUG;
    static constexpr int OFF_PAIR = OFF_DO + Q_STAGES * TILE;
    static constexpr int OFF_P = OFF_PAIR + PAIR_SLOTS * HALF_BYTES;
    static constexpr int OFF_DT = OFF_P + PT_BYTES;
    static constexpr int OFF_MASK = OFF_DT + PT_BYTES;  // [2][128] f32: (mask - c) log2(e) per key
    // per softmax warp: 32 rows x 32 fp32 of dT (128 B rows, 128 B swizzle),
    // added to dpair by one TMA tile reduction
    static constexpr int STG_WARP = 32 * 128;
    static constexpr int OFF_STG = OFF_MASK + 2 * kBN * 4;
    // per dQ warp: 32 rows x 16 fp32 of dQ (64 B rows, 64 B swizzle), added to
    // the fp32 dQ sums by TMA tile reductions, 16 columns at a time
    static constexpr int QSTG_WARP = 32 * 64;
    static constexpr int OFF_QSTG = OFF_STG + (HAS_PAIR ? 4 * GROUPS * STG_WARP : 0);
    static constexpr int OFF_BAR = OFF_QSTG + 4 * QSTG_WARP;
    static constexpr int BAR_KVF = 0;                            // [KV_STAGES] K, V landed
    static constexpr int BAR_KVE = BAR_KVF + KV_STAGES;          // [KV_STAGES] last MMA of the unit done
    static constexpr int BAR_QF = BAR_KVE + KV_STAGES;           // [2] Q, dO landed
    static constexpr int BAR_QE = BAR_QF + Q_STAGES;             // [2] MMAs reading them done
    static constexpr int BAR_BF = BAR_QE + Q_STAGES;             // [PAIR_RING] bias half tile landed
    static constexpr int BAR_BE = BAR_BF + PAIR_RING;            // [PAIR_RING] read by its 4 softmax warps
    static constexpr int BAR_SF = BAR_BE + PAIR_RING;            // S, dP in tensor memory
    static constexpr int BAR_SE = BAR_SF + 1;                    // S, dP read
    static constexpr int BAR_PF = BAR_SE + 1;                    // P, dT tiles written
    static constexpr int BAR_PE = BAR_PF + 1;                    // P, dT tiles read by the MMAs
    static constexpr int BAR_DQF = BAR_PE + 1;                   // dQ in tensor memory
    static constexpr int BAR_DQE = BAR_DQF + 1;                  // dQ read
    static constexpr int BAR_UF = BAR_DQE + 1;                   // dK, dV of a unit final
    static constexpr int BAR_UE = BAR_UF + 1;                    // dK, dV read
    static constexpr int BAR_MKF = BAR_UE + 1;                   // [2] mask row of a unit written
    static constexpr int BAR_DRAIN = BAR_MKF + 2;
    static constexpr int NUM_BARS = BAR_DRAIN + 1;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;      // tmem slot, abort flag
    static constexpr int USED = OFF_MISC + 16;
    static constexpr int SMEM_BYTES = (USED + 1024 > 116 * 1024) ? USED + 1024 : 116 * 1024;
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
    // tensor-memory columns
    static constexpr uint32_t TM_S = 0;
    static constexpr uint32_t TM_DP = 128;
    static constexpr uint32_t TM_DV = 256;
    static constexpr uint32_t TM_DK = TM_DV + ((D + 31) / 32) * 32;          // D + 16 columns
    static constexpr uint32_t TM_DQ = TM_DK + ((D + 16 + 31) / 32) * 32;
    static constexpr uint32_t TMEM_COLS = 512;
    static_assert(TM_DQ + D <= TMEM_COLS, "tensor memory");
    // instruction descriptors: fp32 accumulate, M = 128; operand type bf16
    // (1) or fp16 (0); bit 15 / 16: A / B MN-major
    static constexpr uint32_t AB = F16 ? 0u : ((1u << 7) | (1u << 10));
    static constexpr uint32_t IDESC_S = (1u << 4) | AB | ((uint32_t(kBN) >> 3) << 17) | ((uint32_t(kBM) >> 4) << 24);
    static constexpr uint32_t IDESC_DV =
        (1u << 4) | AB | (1u << 15) | (1u << 16) | ((uint32_t(D) >> 3) << 17) | ((uint32_t(kBM) >> 4) << 24);
    static constexpr uint32_t IDESC_DK =
        (1u << 4) | AB | (1u << 15) | (1u << 16) | ((uint32_t(D + 16) >> 3) << 17) | ((uint32_t(kBM) >> 4) << 24);
    static constexpr uint32_t IDESC_DQ =
        (1u << 4) | AB | (1u << 16) | ((uint32_t(D) >> 3) << 17) | ((uint32_t(kBM) >> 4) << 24);
    static constexpr uint32_t ONE = F16 ? 0x3C00u : 0x3F80u;  // 1.0 in the operand type
};

struct BwdUnit {
    int kb, h, n, b;
    long long bn;
};

__device__ __forceinline__ BwdUnit bwd_unit(const BwdTriParams& p, int u) {
    BwdUnit t;
    t.kb = u % p.num_kb;
    int r = u / p.num_kb;
    t.h = r % p.H;
    r /= p.H;
    t.n = r % p.N;
    t.b = r / p.N;
    t.bn = (long long)t.b * p.N + t.n;
    return t;
}

__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}

template <bool F16>
__device__ __forceinline__ float bits_to_f32(uint32_t bits) {
    if constexpr (F16) return __half2float(__ushort_as_half(uint16_t(bits)));
    else return __uint_as_float(bits << 16);
}

template <bool F16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    if constexpr (F16) return ptx::pack_f16x2(lo, hi);
    else return ptx::pack_bf16x2(lo, hi);
}

template <int D, bool HAS_PAIR, bool F16>
__global__ void __launch_bounds__(BwdCfg<D, HAS_PAIR, F16>::THREADS, 1)
evo_bwd_tri_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                   const __grid_constant__ CUtensorMap tm_pair, const __grid_constant__ CUtensorMap tm_dpair,
                   const __grid_constant__ CUtensorMap tm_dq, const BwdTriParams p) {
    using C = BwdCfg<D, HAS_PAIR, F16>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = ptx::smem_u32(smem);
    const int warp = __shfl_sync(0xffffffffu, int(threadIdx.x >> 5), 0);
    const int lane = threadIdx.x & 31;
    const int G = gridDim.x;
    const int nqb = p.num_qb;

    auto bar = [&](int i) -> uint32_t { return sb + C::OFF_BAR + 8u * uint32_t(i); };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
    const float* mask_s = reinterpret_cast<const float*>(smem + C::OFF_MASK);

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::KV_STAGES; ++s) {
            ptx::mbar_init(bar(C::BAR_KVF + s), 1);
            ptx::mbar_init(bar(C::BAR_KVE + s), 1);
        }
        for (int s = 0; s < C::Q_STAGES; ++s) {
            ptx::mbar_init(bar(C::BAR_QF + s), 1);
            ptx::mbar_init(bar(C::BAR_QE + s), 1);
        }
        for (int s = 0; s < C::PAIR_RING; ++s) {
            ptx::mbar_init(bar(C::BAR_BF + s), 1);
            ptx::mbar_init(bar(C::BAR_BE + s), 4);
        }
        ptx::mbar_init(bar(C::BAR_SF), 1);
        ptx::mbar_init(bar(C::BAR_SE), 4 * C::GROUPS);
        ptx::mbar_init(bar(C::BAR_PF), 4 * C::GROUPS);
        ptx::mbar_init(bar(C::BAR_PE), 1);
        ptx::mbar_init(bar(C::BAR_DQF), 1);
        ptx::mbar_init(bar(C::BAR_DQE), 4);
        ptx::mbar_init(bar(C::BAR_UF), 1);
        ptx::mbar_init(bar(C::BAR_UE), 4);
        ptx::mbar_init(bar(C::BAR_MKF + 0), 4);
        ptx::mbar_init(bar(C::BAR_MKF + 1), 4);
        ptx::mbar_init(bar(C::BAR_DRAIN), 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 0) {
        // the ones box of each Q stage: column 0 (the first of its 16) = 1
        for (int r = lane; r < C::Q_STAGES * kBM; r += 32) {
            const int st = r / kBM, row = r % kBM;
            const uint32_t box = sb + C::OFF_Q + uint32_t(st * C::QAUG + C::TILE);
            ptx::st_shared_v4(box + swz_chunk<32>(row, 0), make_uint4(C::ONE, 0u, 0u, 0u));
            ptx::st_shared_v4(box + swz_chunk<32>(row, 1), make_uint4(0u, 0u, 0u, 0u));
        }
        ptx::fence_proxy_async_smem();
    }
    if (warp == 1) {
        ptx::tmem_alloc(ptx::smem_u32(tmem_slot), C::TMEM_COLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool aborted = false;
    // With two softmax groups the loader / MMA warpgroup hands registers to the
    // softmax and epilogue warps (inside each role's branch, so that the
    // compiler sees which budget each piece of code runs under).
    if (warp == 0) {
        // ------------------------------------------------------------ loads
        if constexpr (C::GROUPS == 2) ptx::setmaxnreg_dec<C::LOW_REGS>();
        if (lane == 0) {
            ptx::prefetch_tmap(&tm_q);
            ptx::prefetch_tmap(&tm_k);
            ptx::prefetch_tmap(&tm_v);
            ptx::prefetch_tmap(&tm_do);
            if (HAS_PAIR) ptx::prefetch_tmap(&tm_pair);
        }
        int n_kv = 0, n_q = 0, n_b = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < p.num_units && ok; u += G) {
            const BwdUnit t = bwd_unit(p, u);
            const int kvs = n_kv % C::KV_STAGES;
            ok = wait_warp(bar(C::BAR_KVE + kvs), ((n_kv / C::KV_STAGES) & 1) ^ 1, abort_flag);
            if (!ok) break;
            {
                const uint32_t kd = sb + C::OFF_K + uint32_t(kvs * C::TILE);
                const uint32_t vd = sb + C::OFF_V + uint32_t(kvs * C::TILE);
                const int s0 = t.kb * kBN, bn = int(t.bn);
                ptx::tma_load_4d_elect(kd, &tm_k, bar(C::BAR_KVF + kvs), 2 * C::TILE, 0, t.h, s0, bn);
#pragma unroll
                for (int x = 1; x < C::NBOX; ++x)
                    ptx::tma_load_4d_more_elect(kd + x * C::BOX, &tm_k, bar(C::BAR_KVF + kvs), 16 * x, t.h, s0, bn);
#pragma unroll
                for (int x = 0; x < C::NBOX; ++x)
                    ptx::tma_load_4d_more_elect(vd + x * C::BOX, &tm_v, bar(C::BAR_KVF + kvs), 16 * x, t.h, s0, bn);
                ++n_kv;
            }
            for (int qb = 0; qb < nqb; ++qb) {
                const int st = n_q % C::Q_STAGES;
                ok = wait_warp(bar(C::BAR_QE + st), ((n_q / C::Q_STAGES) & 1) ^ 1, abort_flag);
                if (!ok) break;
                const uint32_t qd = sb + C::OFF_Q + uint32_t(st * C::QAUG);
                const uint32_t dd = sb + C::OFF_DO + uint32_t(st * C::TILE);
                const int s0 = qb * kBM, bn = int(t.bn);
                ptx::tma_load_4d_elect(qd, &tm_q, bar(C::BAR_QF + st), 2 * C::TILE, 0, t.h, s0, bn);
#pragma unroll
                for (int x = 1; x < C::NBOX; ++x)
                    ptx::tma_load_4d_more_elect(qd + x * C::BOX, &tm_q, bar(C::BAR_QF + st), 16 * x, t.h, s0, bn);
#pragma unroll
                for (int x = 0; x < C::NBOX; ++x)
                    ptx::tma_load_4d_more_elect(dd + x * C::BOX, &tm_do, bar(C::BAR_QF + st), 16 * x, t.h, s0, bn);
                ++n_q;
                if constexpr (HAS_PAIR) {
                    // the step's two half tiles (keys 0-63, 64-127), each in its ring slot
                    for (int x = 0; x < 2 && ok; ++x) {
                        const int ps = n_b % C::PAIR_RING;
                        ok = wait_warp(bar(C::BAR_BE + ps), ((n_b / C::PAIR_RING) & 1) ^ 1, abort_flag);
                        if (!ok) break;
                        if (lane == 0) {
                            const uint32_t dst = sb + C::OFF_PAIR + uint32_t(ps * C::HALF_BYTES);
                            ptx::mbar_arrive_expect_tx(bar(C::BAR_BF + ps), C::HALF_BYTES);
                            ptx::tma_load_3d(dst, &tm_pair, bar(C::BAR_BF + ps), t.kb * kBN + 64 * x, s0,
                                             t.b * p.H + t.h);
                        }
                        __syncwarp();
                        ++n_b;
                    }
                    if (!ok) break;
                }
            }
        }
        if (!ok) {
            aborted = true;
            // let every copy this warp started land before the CTA exits
            if (lane == 0) {
                // the last load issued into each stage (issue index s, s + R, ...)
                auto drain = [&](int n, int R, int base) {
                    for (int s = 0; s < R; ++s)
                        if (n - 1 >= s) {
                            const int last = s + R * ((n - 1 - s) / R);
                            wait_bounded(bar(base + s), uint32_t(last / R) & 1u, nullptr);
                        }
                };
                drain(n_kv, C::KV_STAGES, C::BAR_KVF);
                drain(n_q, C::Q_STAGES, C::BAR_QF);
                if (HAS_PAIR) drain(n_b, C::PAIR_RING, C::BAR_BF);
            }
            __syncwarp();
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------- MMAs
        if constexpr (C::GROUPS == 2) ptx::setmaxnreg_dec<C::LOW_REGS>();
        struct Step {
            bool valid;
            int g, qb, kvs, uc;
            bool last;
        };
        Step prev = {false, 0, 0, 0, 0, false};
        // dV, dK and dQ of one step (its P and dT are in shared memory)
        auto grads = [&](const Step& s) -> bool {
            if (!wait_warp(bar(C::BAR_PF), uint32_t(s.g) & 1u, abort_flag)) return false;
            if (s.qb == 0 && s.uc > 0 && !wait_warp(bar(C::BAR_UE), uint32_t(s.uc - 1) & 1u, abort_flag))
                return false;
            ptx::tc_fence_after();
            const int st = s.g % C::Q_STAGES;
            const uint32_t qd = sb + C::OFF_Q + uint32_t(st * C::QAUG);
            const uint32_t dd = sb + C::OFF_DO + uint32_t(st * C::TILE);
            const uint32_t kd = sb + C::OFF_K + uint32_t(s.kvs * C::TILE);
            const uint32_t pt = sb + C::OFF_P, dt = sb + C::OFF_DT;
#pragma unroll
            for (int kk = 0; kk < kBM / 16; ++kk)
                ptx::mma_ss_elect(tmem + C::TM_DV, desc_mn_major<128>(pt + kk * 2048, C::PT_ATOM),
                                  desc_mn_major<32>(dd + kk * 512, C::BOX), C::IDESC_DV,
                                  (s.qb > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
            for (int kk = 0; kk < kBM / 16; ++kk)
                ptx::mma_ss_elect(tmem + C::TM_DK, desc_mn_major<128>(dt + kk * 2048, C::PT_ATOM),
                                  desc_mn_major<32>(qd + kk * 512, C::BOX), C::IDESC_DK,
                                  (s.qb > 0 || kk > 0) ? 1u : 0u);
            if (s.g > 0) {
                if (!wait_warp(bar(C::BAR_DQE), uint32_t(s.g - 1) & 1u, abort_flag)) return false;
                ptx::tc_fence_after();
            }
#pragma unroll
            for (int kk = 0; kk < kBN / 16; ++kk)
                ptx::mma_ss_elect(tmem + C::TM_DQ,
                                  desc_k_major<128>(dt + (kk / 4) * C::PT_ATOM + (kk % 4) * 32),
                                  desc_mn_major<32>(kd + kk * 512, C::BOX), C::IDESC_DQ, kk > 0 ? 1u : 0u);
            ptx::mma_commit_elect(bar(C::BAR_DQF));
            ptx::mma_commit_elect(bar(C::BAR_PE));
            ptx::mma_commit_elect(bar(C::BAR_QE + st));
            if (s.last) {
                ptx::mma_commit_elect(bar(C::BAR_UF));
                ptx::mma_commit_elect(bar(C::BAR_KVE + s.kvs));
            }
            return true;
        };
        bool ok = true;
        int uc = 0, g = 0;
        for (int u = blockIdx.x; u < p.num_units && ok; u += G, ++uc) {
            const int kvs = uc % C::KV_STAGES;
            for (int qb = 0; qb < nqb; ++qb, ++g) {
                if (qb == 0) {
                    // one K/V stage: the previous unit's MMAs must finish before its reload
                    if (C::KV_STAGES == 1 && prev.valid) {
                        ok = grads(prev);
                        prev.valid = false;
                        if (!ok) break;
                    }
                    ok = wait_warp(bar(C::BAR_KVF + kvs), uint32_t(uc / C::KV_STAGES) & 1u, abort_flag);
                    if (!ok) break;
                }
                const int st = g % C::Q_STAGES;
                ok = wait_warp(bar(C::BAR_QF + st), uint32_t(g / C::Q_STAGES) & 1u, abort_flag);
                if (ok && g > 0) ok = wait_warp(bar(C::BAR_SE), uint32_t(g - 1) & 1u, abort_flag);
                if (!ok) break;
                ptx::tc_fence_after();
                const uint32_t qd = sb + C::OFF_Q + uint32_t(st * C::QAUG);
                const uint32_t dd = sb + C::OFF_DO + uint32_t(st * C::TILE);
                const uint32_t kd = sb + C::OFF_K + uint32_t(kvs * C::TILE);
                const uint32_t vd = sb + C::OFF_V + uint32_t(kvs * C::TILE);
#pragma unroll
                for (int kk = 0; kk < C::NBOX; ++kk)
                    ptx::mma_ss_elect(tmem + C::TM_S, desc_k_major<32>(qd + kk * C::BOX),
                                      desc_k_major<32>(kd + kk * C::BOX), C::IDESC_S, kk > 0 ? 1u : 0u);
#pragma unroll
                for (int kk = 0; kk < C::NBOX; ++kk)
                    ptx::mma_ss_elect(tmem + C::TM_DP, desc_k_major<32>(dd + kk * C::BOX),
                                      desc_k_major<32>(vd + kk * C::BOX), C::IDESC_S, kk > 0 ? 1u : 0u);
                ptx::mma_commit_elect(bar(C::BAR_SF));
                if (prev.valid) {
                    ok = grads(prev);
                    if (!ok) break;
                }
                prev = {true, g, qb, kvs, uc, qb == nqb - 1};
            }
        }
        if (ok && prev.valid) ok = grads(prev);
        if (!ok) {
            aborted = true;
            // every MMA this warp issued completes before tensor memory is freed
            ptx::mma_commit_elect(bar(C::BAR_DRAIN));
            wait_bounded(bar(C::BAR_DRAIN), 0, nullptr);
            __syncwarp();
        }
    } else if (warp < 4) {
        if constexpr (C::GROUPS == 2) ptx::setmaxnreg_dec<C::LOW_REGS>();
    } else if (warp < C::EPI0) {
        // --------------------------------------------------- P and dT rows
        if constexpr (C::GROUPS == 2) ptx::setmaxnreg_inc<C::HIGH_REGS>();
        // group grp takes the 32-key chunks c0 .. c1 - 1 of every row
        const int grp = (warp - 4) >> 2;
        const int sw = warp - 4;                      // stage of this warp's dpair tiles
        const int c0 = grp * (4 / C::GROUPS), c1 = c0 + 4 / C::GROUPS;
        const int wq = (warp - 4) & 3;
        const int r = 32 * wq + lane;                 // query row in the block; key index for the mask row
        const uint32_t tl = tmem + (uint32_t(32 * wq) << 16);
        float* mask_w = reinterpret_cast<float*>(smem + C::OFF_MASK);
        bool ok = true;
        int uc = 0, g = 0;
        // Global loads are issued one step (rows) or one unit (mask) ahead of
        // their use, so that their latency hides behind a step's work.
        auto row_loads = [&](const BwdUnit& t, int qb, float& lr, float& dl) {
            const int i = qb * kBM + r;
            lr = INFINITY;
            dl = 0.f;
            if (i < p.S) {
                const size_t ri = (size_t(t.bn) * p.H + t.h) * p.S + i;
                lr = __ldg(p.lse_r + ri);
                dl = __ldg(p.delta + ri);
            }
        };
        auto mask_loads = [&](const BwdUnit& t, uint32_t& mbits, float& c) {
            const int j = t.kb * kBN + r;
            mbits = 0u;
            c = 0.f;
            if (grp == 0 && p.mask != nullptr && j < p.S) {
                mbits = p.mask[size_t(t.bn) * p.S + j];
                c = __ldg(p.cmask + t.bn);
            }
        };
        float lr_n = INFINITY, dl_n = 0.f, c_n = 0.f;
        uint32_t mbits_n = 0u;
        if (int(blockIdx.x) < p.num_units) {
            const BwdUnit t0 = bwd_unit(p, blockIdx.x);
            row_loads(t0, 0, lr_n, dl_n);
            mask_loads(t0, mbits_n, c_n);
        }
        for (int u = blockIdx.x; u < p.num_units && ok; u += G, ++uc) {
            const BwdUnit t = bwd_unit(p, u);
            const bool has_next_unit = u + G < p.num_units;
            const BwdUnit tn = bwd_unit(p, has_next_unit ? u + G : u);
            const int mb = uc & 1;
            {
                // this unit's key block of the mask row: (mask - c) log2(e), -inf past S
                // or more than kMaskFloor below c (such a weight is exactly zero)
                const int j = t.kb * kBN + r;
                const uint32_t mbits = mbits_n;
                const float cm = c_n;
                if (has_next_unit) mask_loads(tn, mbits_n, c_n);
                float ml = -INFINITY;
                if (j < p.S) {
                    const float x = (p.mask != nullptr) ? bits_to_f32<F16>(mbits) - cm : 0.f;
                    ml = (x < -kMaskFloor) ? -INFINITY : x * kLog2e;
                }
                // the first group writes the row, every group waits for it
                if (grp == 0) {
                    mask_w[mb * kBN + r] = ml;
                    __syncwarp();
                    ptx::mbar_arrive_elect(bar(C::BAR_MKF + mb));
                }
                ok = wait_warp(bar(C::BAR_MKF + mb), uint32_t(uc >> 1) & 1u, abort_flag);
                if (!ok) break;
            }
            const float* ml2 = mask_s + mb * kBN;
            for (int qb = 0; qb < nqb; ++qb, ++g) {
                const float lr = lr_n, dl = dl_n;
                if (qb + 1 < nqb) row_loads(t, qb + 1, lr_n, dl_n);
                else if (has_next_unit) row_loads(tn, 0, lr_n, dl_n);
                ok = wait_warp(bar(C::BAR_SF), uint32_t(g) & 1u, abort_flag);
                if (!ok) break;
                ptx::tc_fence_after();
                const float lse2 = (lr == INFINITY) ? INFINITY : lr * kLog2e;
                // this step's pair-bias half tiles are numbers 2g (keys 0-63) and 2g + 1 of the ring
                // One 32-key chunk: P and dT packed into pw, dw, its dT tile added to
                // dpair (the reduction needs no wait for the previous step's MMAs, so
                // it is issued before the P and dT stores)
                auto chunk = [&](int c, uint32_t* pw, uint32_t* dw) -> bool {
                    const int hs = (2 * g + (c >> 1)) % C::PAIR_RING;
                    if (HAS_PAIR && (c & 1) == 0) {
                        ok = wait_warp(bar(C::BAR_BF + hs), uint32_t((2 * g + (c >> 1)) / C::PAIR_RING) & 1u,
                                       abort_flag);
                        if (!ok) return false;
                    }
                    float s[32], dp[32];
                    ptx::tmem_ld_x32(tl + C::TM_S + 32u * c, reinterpret_cast<uint32_t*>(s));
                    ptx::tmem_ld_x32(tl + C::TM_DP + 32u * c, reinterpret_cast<uint32_t*>(dp));
                    ptx::tmem_ld_wait_x32(reinterpret_cast<uint32_t*>(s));
                    ptx::reg_fence_x32(reinterpret_cast<uint32_t*>(dp));
                    if (c == c1 - 1) {
                        ptx::tc_fence_before();
                        ptx::mbar_arrive_elect(bar(C::BAR_SE));
                    }
                    // s <- the exponent of p in log2 units, then p; dp <- dT
#pragma unroll
                    for (int q4 = 0; q4 < 8; ++q4) {
                        const float4 m4 = *reinterpret_cast<const float4*>(ml2 + 32 * c + 4 * q4);
                        s[4 * q4 + 0] = fmaf(s[4 * q4 + 0], p.scale_log2, m4.x - lse2);
                        s[4 * q4 + 1] = fmaf(s[4 * q4 + 1], p.scale_log2, m4.y - lse2);
                        s[4 * q4 + 2] = fmaf(s[4 * q4 + 2], p.scale_log2, m4.z - lse2);
                        s[4 * q4 + 3] = fmaf(s[4 * q4 + 3], p.scale_log2, m4.w - lse2);
                    }
                    if constexpr (HAS_PAIR) {
                        const uint32_t base = sb + C::OFF_PAIR + uint32_t(hs * C::HALF_BYTES);
#pragma unroll
                        for (int u4 = 0; u4 < 4; ++u4) {
                            const uint4 w = ptx::ld_shared_v4(base + swz_chunk<128>(r, (c % 2) * 4 + u4));
                            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                s[8 * u4 + 2 * e] = fmaf(bits_to_f32<F16>(ws[e] & 0xffffu), kLog2e, s[8 * u4 + 2 * e]);
                                s[8 * u4 + 2 * e + 1] =
                                    fmaf(bits_to_f32<F16>(ws[e] >> 16), kLog2e, s[8 * u4 + 2 * e + 1]);
                            }
                        }
                    }
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        s[e] = ptx::ex2_approx(s[e]);
                        s[e + 1] = ptx::ex2_approx(s[e + 1]);
                        dp[e] = s[e] * (dp[e] - dl);
                        dp[e + 1] = s[e + 1] * (dp[e + 1] - dl);
                        pw[e / 2] = pack2<F16>(s[e], s[e + 1]);
                        dw[e / 2] = pack2<F16>(dp[e], dp[e + 1]);
                    }
                    if (HAS_PAIR && p.dpair_acc != nullptr) {
                        // this warp's 32 rows x 32 keys of dT, staged in shared memory and
                        // added to dpair by one TMA tile reduction (whole 128 B rows in L2);
                        // lane 0 issues it and first waits until the previous one has
                        // read the stage
                        const uint32_t stg = sb + C::OFF_STG + uint32_t(sw * C::STG_WARP);
                        if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
                        __syncwarp();
#pragma unroll
                        for (int q4 = 0; q4 < 8; ++q4)
                            ptx::st_shared_v4(stg + swz_chunk<128>(lane, q4),
                                              make_uint4(__float_as_uint(dp[4 * q4]), __float_as_uint(dp[4 * q4 + 1]),
                                                         __float_as_uint(dp[4 * q4 + 2]), __float_as_uint(dp[4 * q4 + 3])));
                        ptx::fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            asm volatile(
                                "cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.tile.bulk_group"
                                " [%0, {%2, %3, %4}], [%1];" ::"l"(reinterpret_cast<uint64_t>(&tm_dpair)),
                                "r"(stg), "r"(t.kb * kBN + 32 * c), "r"(qb * kBM + 32 * wq), "r"(t.b * p.H + t.h)
                                : "memory");
                            asm volatile("cp.async.bulk.commit_group;" ::: "memory");
                        }
                    }
                    if (HAS_PAIR && (c & 1) == 1) {
                        // the last chunk of this half tile has read it
                        __syncwarp();
                        ptx::mbar_arrive_elect(bar(C::BAR_BE + hs));
                    }
                    return true;
                };
                auto store = [&](int c, const uint32_t* pw, const uint32_t* dw) {
                    const uint32_t poff = uint32_t((c / 2) * C::PT_ATOM);
#pragma unroll
                    for (int u4 = 0; u4 < 4; ++u4) {
                        const uint32_t off = poff + swz_chunk<128>(r, (c % 2) * 4 + u4);
                        ptx::st_shared_v4(sb + C::OFF_P + off,
                                          make_uint4(pw[4 * u4], pw[4 * u4 + 1], pw[4 * u4 + 2], pw[4 * u4 + 3]));
                        ptx::st_shared_v4(sb + C::OFF_DT + off,
                                          make_uint4(dw[4 * u4], dw[4 * u4 + 1], dw[4 * u4 + 2], dw[4 * u4 + 3]));
                    }
                };
                if constexpr (C::GROUPS == 2) {
                    // both chunks first (they overlap the previous step's MMAs), then
                    // the wait for those MMAs to have read the P and dT tiles
                    uint32_t pwa[16], dwa[16], pwb[16], dwb[16];
                    ok = chunk(c0, pwa, dwa) && chunk(c0 + 1, pwb, dwb);
                    if (ok && g > 0) ok = wait_warp(bar(C::BAR_PE), uint32_t(g - 1) & 1u, abort_flag);
                    if (!ok) break;
                    store(c0, pwa, dwa);
                    store(c0 + 1, pwb, dwb);
                } else {
#pragma unroll 1
                    for (int c = c0; c < c1; ++c) {
                        uint32_t pw[16], dw[16];
                        if (!(ok = chunk(c, pw, dw))) break;
                        if (c == c0 && g > 0) {
                            // the MMAs of the previous step have read the P and dT tiles
                            ok = wait_warp(bar(C::BAR_PE), uint32_t(g - 1) & 1u, abort_flag);
                            if (!ok) break;
                        }
                        store(c, pw, dw);
                    }
                }
                if (!ok) break;
                ptx::fence_proxy_async_smem();  // generic-proxy writes -> tensor-core reads
                __syncwarp();
                ptx::mbar_arrive_elect(bar(C::BAR_PF));
            }
        }
        // every dpair reduction of this warp has been carried out
        if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
        __syncwarp();
        if (!ok) aborted = true;
    } else {
        // ------------------------------------------- dQ, dK, dV, dmask out
        if constexpr (C::GROUPS == 2) ptx::setmaxnreg_inc<C::HIGH_REGS>();
        const int we = warp - C::EPI0;
        const int r = 32 * we + lane;
        const uint32_t tl = tmem + (uint32_t(32 * we) << 16);
        constexpr int LDW = D >= 32 ? 32 : 16;  // columns per tensor-memory load
        bool ok = true;
        int uc = 0, g = 0;
        for (int u = blockIdx.x; u < p.num_units && ok; u += G, ++uc) {
            const BwdUnit t = bwd_unit(p, u);
            for (int qb = 0; qb < nqb; ++qb, ++g) {
                ok = wait_warp(bar(C::BAR_DQF), uint32_t(g) & 1u, abort_flag);
                if (!ok) break;
                ptx::tc_fence_after();
                float dq[D];
#pragma unroll
                for (int d0 = 0; d0 < D; d0 += LDW) {
                    if constexpr (LDW == 32) ptx::tmem_ld_x32(tl + C::TM_DQ + d0, reinterpret_cast<uint32_t*>(dq + d0));
                    else ptx::tmem_ld_x16(tl + C::TM_DQ + d0, reinterpret_cast<uint32_t*>(dq + d0));
                }
                if constexpr (LDW == 32) ptx::tmem_ld_wait_x32(reinterpret_cast<uint32_t*>(dq));
                else ptx::tmem_ld_wait_x16(reinterpret_cast<uint32_t*>(dq));
#pragma unroll
                for (int d0 = LDW; d0 < D; d0 += 32) ptx::reg_fence_x32(reinterpret_cast<uint32_t*>(dq + d0));
                ptx::tc_fence_before();
                ptx::mbar_arrive_elect(bar(C::BAR_DQE));
                // this warp's 32 rows of dQ into the fp32 sums, 16 columns per TMA
                // tile reduction (rows past S are clipped by the tensor map)
                const uint32_t stg = sb + C::OFF_QSTG + uint32_t(we * C::QSTG_WARP);
#pragma unroll
                for (int x = 0; x < D / 16; ++x) {
                    if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
                    __syncwarp();
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        ptx::st_shared_v4(stg + swz_chunk<64>(lane, q4),
                                          make_uint4(__float_as_uint(dq[16 * x + 4 * q4]),
                                                     __float_as_uint(dq[16 * x + 4 * q4 + 1]),
                                                     __float_as_uint(dq[16 * x + 4 * q4 + 2]),
                                                     __float_as_uint(dq[16 * x + 4 * q4 + 3])));
                    ptx::fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        asm volatile(
                            "cp.reduce.async.bulk.tensor.4d.global.shared::cta.add.tile.bulk_group"
                            " [%0, {%2, %3, %4, %5}], [%1];" ::"l"(reinterpret_cast<uint64_t>(&tm_dq)),
                            "r"(stg), "r"(16 * x), "r"(t.h), "r"(qb * kBM + 32 * we), "r"(int(t.bn))
                            : "memory");
                        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
                    }
                }
            }
            if (!ok) break;
            // the unit's dK, dV (and this head's dmask share) are final
            ok = wait_warp(bar(C::BAR_UF), uint32_t(uc) & 1u, abort_flag);
            if (!ok) break;
            ptx::tc_fence_after();
            float acc[D];
            uint32_t vpk[D / 2];
#pragma unroll
            for (int d0 = 0; d0 < D; d0 += LDW) {
                if constexpr (LDW == 32) ptx::tmem_ld_x32(tl + C::TM_DV + d0, reinterpret_cast<uint32_t*>(acc + d0));
                else ptx::tmem_ld_x16(tl + C::TM_DV + d0, reinterpret_cast<uint32_t*>(acc + d0));
            }
            if constexpr (LDW == 32) ptx::tmem_ld_wait_x32(reinterpret_cast<uint32_t*>(acc));
            else ptx::tmem_ld_wait_x16(reinterpret_cast<uint32_t*>(acc));
#pragma unroll
            for (int d0 = LDW; d0 < D; d0 += 32) ptx::reg_fence_x32(reinterpret_cast<uint32_t*>(acc + d0));
#pragma unroll
            for (int d = 0; d < D; d += 2) vpk[d / 2] = pack2<F16>(acc[d], acc[d + 1]);
            float dka[D + 16];
#pragma unroll
            for (int d0 = 0; d0 < D + 16; d0 += 16)
                ptx::tmem_ld_x16(tl + C::TM_DK + d0, reinterpret_cast<uint32_t*>(dka + d0));
            ptx::tmem_ld_wait_x16(reinterpret_cast<uint32_t*>(dka));
#pragma unroll
            for (int d0 = 16; d0 < D + 16; d0 += 16) {
                uint32_t* rr = reinterpret_cast<uint32_t*>(dka + d0);
                ptx::reg_fence_x8(rr);
                ptx::reg_fence_x8(rr + 8);
            }
            ptx::tc_fence_before();
            ptx::mbar_arrive_elect(bar(C::BAR_UE));
            const int j = t.kb * kBN + r;
            if (j < p.S) {
                const size_t off = ((size_t(t.bn) * p.S + j) * p.H + t.h) * D;
                uint4* kdst = reinterpret_cast<uint4*>(p.dk + off);
                uint4* vdst = reinterpret_cast<uint4*>(p.dv + off);
#pragma unroll
                for (int d = 0; d < D; d += 8) {
                    kdst[d / 8] = make_uint4(pack2<F16>(dka[d] * p.scale, dka[d + 1] * p.scale),
                                             pack2<F16>(dka[d + 2] * p.scale, dka[d + 3] * p.scale),
                                             pack2<F16>(dka[d + 4] * p.scale, dka[d + 5] * p.scale),
                                             pack2<F16>(dka[d + 6] * p.scale, dka[d + 7] * p.scale));
                    vdst[d / 8] = make_uint4(vpk[d / 2], vpk[d / 2 + 1], vpk[d / 2 + 2], vpk[d / 2 + 3]);
                }
                if (p.dmask_acc != nullptr) atomicAdd(p.dmask_acc + size_t(t.bn) * p.S + j, dka[D]);
            }
        }
        // every dQ reduction of this warp has been carried out
        if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
        __syncwarp();
        if (!ok) aborted = true;
    }
    (void)aborted;

    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == 1) ptx::tmem_dealloc(tmem, C::TMEM_COLS);
}

// Rounds the fp32 sums of the tensor-core backward to the output type: dQ
// (times 1 / sqrt(D)), and dmask, dpair where requested.
template <bool F16>
__global__ void __launch_bounds__(256) evo_bwd_post_kernel(const float* dq_acc, uint16_t* dq, long long n_q,
                                                           float scale, const float* dmask_acc, uint16_t* dmask,
                                                           long long n_m, const float* dpair_acc, uint16_t* dpair,
                                                           long long n_p) {
    const long long stride = (long long)gridDim.x * blockDim.x;
    const long long t0 = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    auto cvt = [](float x) -> uint16_t {
        if constexpr (F16) return __half_as_ushort(__float2half_rn(x));
        else return __bfloat16_as_ushort(__float2bfloat16_rn(x));
    };
    // n_q is a multiple of 16 (D is)
    for (long long i = t0; i < n_q / 4; i += stride) {
        const float4 v = reinterpret_cast<const float4*>(dq_acc)[i];
        uint2 o;
        o.x = pack2<F16>(v.x * scale, v.y * scale);
        o.y = pack2<F16>(v.z * scale, v.w * scale);
        reinterpret_cast<uint2*>(dq)[i] = o;
    }
    if (dmask != nullptr)
        for (long long i = t0; i < n_m; i += stride) dmask[i] = cvt(dmask_acc[i]);
    if (dpair != nullptr)
        for (long long i = t0; i < n_p; i += stride) dpair[i] = cvt(dpair_acc[i]);
}

}  // namespace evo
