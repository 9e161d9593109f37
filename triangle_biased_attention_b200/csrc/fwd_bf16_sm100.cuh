// bf16 biased-attention forward on sm_100a: TMA -> tcgen05 MMA into tensor
// memory -> online exp2 softmax in registers -> tcgen05 MMA for P.V.
//
// What it computes is the forward pass of the DeepSpeed DS4Sci_EvoformerAttention
// guide (hmyw.cn): section 4's reference softmax(Q K^T * scale + biases) V,
// with section 5.2's bias shapes and section 5.4's log-sum-exp; the guide's
// own kernel is a CUTLASS fused GEMM + softmax (section 1) written for sm70 to
// sm80-class parts.  This kernel is designed for Blackwell instead:
//
//  * One CTA owns one (b, h, 128-query block) and TWO n slices, n0 and n0+1.
//    The pair bias [B,1,H,S,S] does not depend on n, so both slices read the
//    same 128x128 bias tile from shared memory: one L2->SM transfer feeds two
//    softmax warpgroups.
//  * Warp roles (384 threads): warp 0 issues TMA loads (Q once; K, V and bias
//    tiles through rings of mbarrier-tracked stages); warp 1 issues tcgen05
//    MMAs from one thread; warp 2 turns the mask row into a log2-scaled fp32
//    vector per key block (and computes the per-(b,n) rebase, below); warps
//    4-7 and 8-11 are the softmax warpgroups of slice n0 and n0+1.  Thread r of
//    a warpgroup owns query row r, which is TMEM lane r, so row max and row sum
//    stay in one thread.
//  * Tensor memory (512 columns): per slice, S = Q K^T (128 fp32 columns),
//    P = softmax numerators as bf16 (64 columns) and the O accumulator
//    (D columns).  S and P are separate so the next block's Q K^T can start as
//    soon as the softmax has pulled S into registers.
//  * Online softmax in base 2: u = s*log2(e)/sqrt(D) + (pair + mask - c)*log2(e),
//    p = 2^(u - m).  The running maximum m is only moved when the block maximum
//    exceeds it by more than 8 (p <= 256, exact after the final division by
//    the row sum); moving it rescales O in tensor memory.
//  * Mask rebase: c[b,n] = max_j mask[b,n,j] is subtracted from the mask and
//    added back to the LSE.  The guide builds masks as 1e9*(mask-1) (section
//    5.2); for an n whose every key is masked that is a constant shift of the
//    row, and the rebase keeps fp32 from rounding every logit to -1e9.
//  * Every wait is bounded (about two seconds); on expiry the CTA records
//    EVO_ERR_TIMEOUT, drains its own in-flight copies and MMAs, frees tensor
//    memory and exits.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "common.cuh"
#include "ptx_sm100.cuh"

namespace evo {

struct Bf16Params {
    const uint16_t* mask;  // [B, N, S] bf16 bits, or nullptr
    uint16_t* out;         // [B, N, S, H, D] bf16 bits
    float* lse;            // [B, N, H, S]
    int N, S, H;
    int num_kb;            // key blocks of 128
    float scale_log2;      // log2(e) / sqrt(D)
};

constexpr int kBM = 128;          // query rows per slice tile
constexpr int kBN = 128;          // keys per block
constexpr int kThreads = 384;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: p <= 2^8 between rescales

// UMMA shared-memory descriptor layout codes for swizzle spans of 32/64/128 B.
__host__ __device__ constexpr uint32_t umma_layout_code(int sw_bytes) {
    return sw_bytes == 128 ? 2u : (sw_bytes == 64 ? 4u : 6u);
}

template <int D, bool HAS_PAIR>
struct Bf16Cfg {
    static_assert(D == 16 || D == 32 || D == 64, "head dim");
    static constexpr int ROW = D * 2;                 // bytes per Q/K/V row = swizzle span
    static constexpr int TILE = kBM * ROW;            // one Q, K or V tile
    static constexpr int K_STAGES = (D <= 32) ? 4 : 3;
    static constexpr int V_STAGES = (D <= 32) ? 4 : 3;
    static constexpr int B_STAGES = HAS_PAIR ? 2 : 0;
    static constexpr int M_STAGES = 2;
    static constexpr int BIAS_BYTES = kBM * kBN * 2;  // two 128x64 boxes, 128 B swizzle
    // shared-memory map (offsets from a 1024-aligned base)
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + 2 * TILE;
    static constexpr int OFF_V = OFF_K + K_STAGES * TILE;
    static constexpr int OFF_BIAS = OFF_V + V_STAGES * TILE;
    static constexpr int OFF_MASK = OFF_BIAS + B_STAGES * BIAS_BYTES;  // [2][M_STAGES][128] f32
    static constexpr int OFF_BAR = OFF_MASK + 2 * M_STAGES * kBN * 4;
    // barrier indices
    static constexpr int BAR_Q = 0;
    static constexpr int BAR_KF = 1;
    static constexpr int BAR_KE = BAR_KF + K_STAGES;
    static constexpr int BAR_VF = BAR_KE + K_STAGES;
    static constexpr int BAR_VE = BAR_VF + V_STAGES;
    static constexpr int BAR_BF = BAR_VE + V_STAGES;
    static constexpr int BAR_BE = BAR_BF + 2;
    static constexpr int BAR_MF = BAR_BE + 2;           // [2][M_STAGES]
    static constexpr int BAR_ME = BAR_MF + 2 * M_STAGES;
    static constexpr int BAR_SF = BAR_ME + 2 * M_STAGES;  // [2]
    static constexpr int BAR_SE = BAR_SF + 2;
    static constexpr int BAR_PF = BAR_SE + 2;
    static constexpr int BAR_PE = BAR_PF + 2;
    static constexpr int BAR_DRAIN = BAR_PE + 2;
    static constexpr int NUM_BARS = BAR_DRAIN + 1;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;  // tmem slot, abort flag, c[2]
    static constexpr int USED = OFF_MISC + 16;
    // Request at least 116 KB so that two CTAs never share an SM: each CTA
    // allocates all 512 tensor-memory columns.
    static constexpr int SMEM_BYTES = (USED + 1024 > 116 * 1024) ? USED + 1024 : 116 * 1024;
    static_assert(USED + 1024 <= 227 * 1024, "shared memory");
    // tensor-memory columns
    static constexpr uint32_t TM_S0 = 0;    // + 128 * w
    static constexpr uint32_t TM_P0 = 256;  // + 64 * w
    static constexpr uint32_t TM_O0 = 384;  // + D * w
    static constexpr uint32_t TMEM_COLS = 512;
    // instruction descriptors: fp32 accumulate, bf16 A and B, M = 128
    static constexpr uint32_t IDESC_QK =
        (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t(kBN) >> 3) << 17) | ((uint32_t(kBM) >> 4) << 24);
    static constexpr uint32_t IDESC_PV = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                                         ((uint32_t(D) >> 3) << 17) | ((uint32_t(kBM) >> 4) << 24);
};

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

// MN-major operand tile (V as the B operand of P.V: N = D contiguous, K = keys
// along rows): one swizzle atom spans all D columns; 8-key groups ROW*8 apart.
template <int ROW>
__device__ __forceinline__ uint64_t desc_mn_major(uint32_t saddr, uint32_t tile_bytes) {
    uint64_t d = 0;
    d |= uint64_t((saddr >> 4) & 0x3FFFu);
    d |= uint64_t((tile_bytes >> 4) & 0x3FFFu) << 16;        // next MN atom (none here)
    d |= uint64_t(((8u * ROW) >> 4) & 0x3FFFu) << 32;        // stride between 8-key groups
    d |= uint64_t(1) << 46;
    d |= uint64_t(umma_layout_code(ROW)) << 61;
    return d;
}

template <int D, bool HAS_PAIR>
__global__ void __launch_bounds__(kThreads, 1)
evo_fwd_bf16_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_pair,
                    const Bf16Params p) {
    using C = Bf16Cfg<D, HAS_PAIR>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = ptx::smem_u32(smem);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * 2;
    const int q0 = blockIdx.y * kBM;
    const int bh = blockIdx.z;
    const int b = bh / p.H;
    const int h = bh - b * p.H;
    const int n_valid = (p.N - n0) < 2 ? (p.N - n0) : 2;
    const int nkb = p.num_kb;

    auto bar = [&](int i) -> uint32_t { return sb + C::OFF_BAR + 8u * uint32_t(i); };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
    float* csub_s = reinterpret_cast<float*>(smem + C::OFF_MISC + 8);

    if (threadIdx.x == 0) {
        ptx::mbar_init(bar(C::BAR_Q), 1);
        for (int s = 0; s < C::K_STAGES; ++s) {
            ptx::mbar_init(bar(C::BAR_KF + s), 1);
            ptx::mbar_init(bar(C::BAR_KE + s), 1);
        }
        for (int s = 0; s < C::V_STAGES; ++s) {
            ptx::mbar_init(bar(C::BAR_VF + s), 1);
            ptx::mbar_init(bar(C::BAR_VE + s), 1);
        }
        for (int s = 0; s < 2; ++s) {
            ptx::mbar_init(bar(C::BAR_BF + s), 1);
            ptx::mbar_init(bar(C::BAR_BE + s), 4 * n_valid);
        }
        for (int s = 0; s < 2 * C::M_STAGES; ++s) {
            ptx::mbar_init(bar(C::BAR_MF + s), 32);
            ptx::mbar_init(bar(C::BAR_ME + s), 4);
        }
        for (int w = 0; w < 2; ++w) {
            ptx::mbar_init(bar(C::BAR_SF + w), 1);
            ptx::mbar_init(bar(C::BAR_SE + w), 4);
            ptx::mbar_init(bar(C::BAR_PF + w), 4);
            ptx::mbar_init(bar(C::BAR_PE + w), 1);
        }
        ptx::mbar_init(bar(C::BAR_DRAIN), 1);
        *abort_flag = 0;
        csub_s[0] = 0.f;
        csub_s[1] = 0.f;
        ptx::fence_mbar_init();
    }
    if (warp == 0) {
        ptx::tmem_alloc(ptx::smem_u32(tmem_slot), C::TMEM_COLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            ptx::prefetch_tmap(&tm_q);
            ptx::prefetch_tmap(&tm_k);
            ptx::prefetch_tmap(&tm_v);
            if (HAS_PAIR) ptx::prefetch_tmap(&tm_pair);
            const int bn0 = b * p.N + n0;
            ptx::mbar_arrive_expect_tx(bar(C::BAR_Q), uint32_t(n_valid * C::TILE));
            for (int w = 0; w < n_valid; ++w)
                ptx::tma_load_4d(sb + C::OFF_Q + w * C::TILE, &tm_q, bar(C::BAR_Q), 0, h, q0, bn0 + w);
            int k_issued = 0, v_issued = 0, b_issued = 0;
            bool ok = true;
            for (int j = 0; j < nkb && ok; ++j) {
                for (int w = 0; w < n_valid && ok; ++w) {
                    const int s = k_issued % C::K_STAGES;
                    const uint32_t ph = (k_issued / C::K_STAGES) & 1;
                    if (!wait_bounded(bar(C::BAR_KE + s), ph ^ 1, abort_flag)) { ok = false; break; }
                    ptx::mbar_arrive_expect_tx(bar(C::BAR_KF + s), C::TILE);
                    ptx::tma_load_4d(sb + C::OFF_K + s * C::TILE, &tm_k, bar(C::BAR_KF + s), 0, h, j * kBN, bn0 + w);
                    ++k_issued;
                }
                if (HAS_PAIR && ok) {
                    const int s = b_issued % 2;
                    const uint32_t ph = (b_issued / 2) & 1;
                    if (!wait_bounded(bar(C::BAR_BE + s), ph ^ 1, abort_flag)) { ok = false; break; }
                    const uint32_t dst = sb + C::OFF_BIAS + s * C::BIAS_BYTES;
                    ptx::mbar_arrive_expect_tx(bar(C::BAR_BF + s), C::BIAS_BYTES);
                    ptx::tma_load_3d(dst, &tm_pair, bar(C::BAR_BF + s), j * kBN, q0, bh);
                    ptx::tma_load_3d(dst + C::BIAS_BYTES / 2, &tm_pair, bar(C::BAR_BF + s), j * kBN + 64, q0, bh);
                    ++b_issued;
                }
                for (int w = 0; w < n_valid && ok; ++w) {
                    const int s = v_issued % C::V_STAGES;
                    const uint32_t ph = (v_issued / C::V_STAGES) & 1;
                    if (!wait_bounded(bar(C::BAR_VE + s), ph ^ 1, abort_flag)) { ok = false; break; }
                    ptx::mbar_arrive_expect_tx(bar(C::BAR_VF + s), C::TILE);
                    ptx::tma_load_4d(sb + C::OFF_V + s * C::TILE, &tm_v, bar(C::BAR_VF + s), 0, h, j * kBN, bn0 + w);
                    ++v_issued;
                }
            }
            if (!ok) {
                // Let every copy this thread started land before the CTA exits.
                wait_bounded(bar(C::BAR_Q), 0, nullptr);
                for (int i = (k_issued > C::K_STAGES ? k_issued - C::K_STAGES : 0); i < k_issued; ++i)
                    wait_bounded(bar(C::BAR_KF + i % C::K_STAGES), (i / C::K_STAGES) & 1, nullptr);
                for (int i = (v_issued > C::V_STAGES ? v_issued - C::V_STAGES : 0); i < v_issued; ++i)
                    wait_bounded(bar(C::BAR_VF + i % C::V_STAGES), (i / C::V_STAGES) & 1, nullptr);
                for (int i = (b_issued > 2 ? b_issued - 2 : 0); i < b_issued; ++i)
                    wait_bounded(bar(C::BAR_BF + i % 2), (i / 2) & 1, nullptr);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------- MMA issuer
        if (lane == 0) {
            bool ok = wait_bounded(bar(C::BAR_Q), 0, abort_flag);
            ptx::tc_fence_after();
            int k_used = 0, v_used = 0;
            auto issue_qk = [&](int w) -> bool {
                const int s = k_used % C::K_STAGES;
                if (!wait_bounded(bar(C::BAR_KF + s), (k_used / C::K_STAGES) & 1, abort_flag)) return false;
                ptx::tc_fence_after();
                const uint64_t a = desc_k_major<C::ROW>(sb + C::OFF_Q + w * C::TILE);
                const uint64_t bdesc = desc_k_major<C::ROW>(sb + C::OFF_K + s * C::TILE);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)  // 16 bf16 = 32 B per K step
                    ptx::mma_ss(tmem + C::TM_S0 + 128u * w, a + uint64_t(2 * kk), bdesc + uint64_t(2 * kk),
                                C::IDESC_QK, kk > 0 ? 1u : 0u);
                ptx::mma_commit(bar(C::BAR_KE + s));
                ptx::mma_commit(bar(C::BAR_SF + w));
                ++k_used;
                return true;
            };
            for (int w = 0; w < n_valid && ok; ++w) ok = issue_qk(w);
            for (int j = 0; j < nkb && ok; ++j) {
                if (j + 1 < nkb) {
                    for (int w = 0; w < n_valid && ok; ++w) {
                        ok = wait_bounded(bar(C::BAR_SE + w), j & 1, abort_flag) && issue_qk(w);
                    }
                }
                for (int w = 0; w < n_valid && ok; ++w) {
                    const int s = v_used % C::V_STAGES;
                    ok = wait_bounded(bar(C::BAR_VF + s), (v_used / C::V_STAGES) & 1, abort_flag) &&
                         wait_bounded(bar(C::BAR_PF + w), j & 1, abort_flag);
                    if (!ok) break;
                    ptx::tc_fence_after();
                    const uint64_t bdesc = desc_mn_major<C::ROW>(sb + C::OFF_V + s * C::TILE, C::TILE);
#pragma unroll
                    for (int kk = 0; kk < kBN / 16; ++kk)  // 16 keys per K step = 16 rows of V
                        ptx::mma_ts(tmem + C::TM_O0 + uint32_t(D) * w, tmem + C::TM_P0 + 64u * w + 8u * kk,
                                    bdesc + uint64_t((16 * C::ROW * kk) >> 4), C::IDESC_PV,
                                    (j > 0 || kk > 0) ? 1u : 0u);
                    ptx::mma_commit(bar(C::BAR_VE + s));
                    ptx::mma_commit(bar(C::BAR_PE + w));
                    ++v_used;
                }
            }
            if (!ok) {
                // Wait for every MMA this thread issued before tensor memory is freed.
                ptx::mma_commit(bar(C::BAR_DRAIN));
                wait_bounded(bar(C::BAR_DRAIN), 0, nullptr);
            }
        }
        __syncwarp();
    } else if (warp == 2) {
        // ---------------------------------------------------------- mask warp
        float csub[2] = {0.f, 0.f};
        const uint16_t* mrow[2] = {nullptr, nullptr};
        for (int w = 0; w < n_valid; ++w) {
            if (p.mask != nullptr) {
                mrow[w] = p.mask + (size_t(b) * p.N + n0 + w) * size_t(p.S);
                float mx = -INFINITY;
                for (int j = lane; j < p.S; j += 32) mx = fmaxf(mx, __uint_as_float(uint32_t(mrow[w][j]) << 16));
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                csub[w] = (mx == -INFINITY) ? 0.f : mx;  // all -inf: leave -inf logits, LSE = -inf
            }
            if (lane == 0) csub_s[w] = csub[w];
        }
        bool ok = true;
        for (int j = 0; j < nkb && ok; ++j) {
            for (int w = 0; w < n_valid && ok; ++w) {
                const int stage = j % C::M_STAGES;
                const uint32_t ph = (j / C::M_STAGES) & 1;
                if (!wait_warp(bar(C::BAR_ME + w * C::M_STAGES + stage), ph ^ 1, abort_flag)) { ok = false; break; }
                float* dst = reinterpret_cast<float*>(smem + C::OFF_MASK) + (w * C::M_STAGES + stage) * kBN;
#pragma unroll
                for (int t = lane; t < kBN; t += 32) {
                    const int key = j * kBN + t;
                    float v = -INFINITY;
                    if (key < p.S) {
                        const float m = mrow[w] ? __uint_as_float(uint32_t(mrow[w][key]) << 16) : 0.f;
                        v = (m - csub[w]) * kLog2e;
                    }
                    dst[t] = v;
                }
                ptx::mbar_arrive(bar(C::BAR_MF + w * C::M_STAGES + stage));
            }
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ------------------------------------------------------------ softmax
        const int w = (warp - 4) >> 2;
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;  // query row in the tile == TMEM lane
        if (w < n_valid) {
            const uint32_t lane_base = uint32_t(quarter * 32) << 16;
            const uint32_t tS = tmem + lane_base + C::TM_S0 + 128u * w;
            const uint32_t tP = tmem + lane_base + C::TM_P0 + 64u * w;
            const uint32_t tO = tmem + lane_base + C::TM_O0 + uint32_t(D) * w;
            float m_used = -INFINITY;
            float l = 0.f;
            bool ok = true;
            for (int j = 0; j < nkb; ++j) {
                uint32_t s[128];
                ok = wait_warp(bar(C::BAR_SF + w), j & 1, abort_flag);
                if (!ok) break;
                ptx::tc_fence_after();
                ptx::tmem_ld_x32(tS + 0, s);
                ptx::tmem_ld_x32(tS + 32, s + 32);
                ptx::tmem_ld_x32(tS + 64, s + 64);
                ptx::tmem_ld_x32(tS + 96, s + 96);
                ptx::tmem_ld_wait_x32(s);
                ptx::reg_fence_x32(s + 32);
                ptx::reg_fence_x32(s + 64);
                ptx::reg_fence_x32(s + 96);
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(bar(C::BAR_SE + w));

                const int mstage = j % C::M_STAGES;
                ok = wait_warp(bar(C::BAR_MF + w * C::M_STAGES + mstage), (j / C::M_STAGES) & 1, abort_flag);
                if (!ok) break;
                const int bstage = j & 1;
                if (HAS_PAIR) {
                    ok = wait_warp(bar(C::BAR_BF + bstage), (j >> 1) & 1, abort_flag);
                    if (!ok) break;
                }
                const uint32_t maddr = sb + C::OFF_MASK + uint32_t((w * C::M_STAGES + mstage) * kBN * 4);
                const uint32_t brow = sb + C::OFF_BIAS + uint32_t(bstage * C::BIAS_BYTES) + uint32_t(r * 128);
                float rmax = -INFINITY;
#pragma unroll
                for (int cc = 0; cc < 16; ++cc) {  // 8 keys per step
                    const float4 m0 = ptx::ld_shared_f4(maddr + cc * 32);
                    const float4 m1 = ptx::ld_shared_f4(maddr + cc * 32 + 16);
                    float bias[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
                    if (HAS_PAIR) {
                        // 128 B swizzle: 16 B chunk c of row r sits at chunk c ^ (r % 8)
                        const int box = cc >> 3, c = cc & 7;
                        const uint4 pw = ptx::ld_shared_v4(brow + uint32_t(box * (C::BIAS_BYTES / 2)) +
                                                           uint32_t(((c ^ (r & 7)) << 4)));
                        const uint32_t wv[4] = {pw.x, pw.y, pw.z, pw.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            bias[2 * e] = fmaf(ptx::bf16lo_to_f32(wv[e]), kLog2e, bias[2 * e]);
                            bias[2 * e + 1] = fmaf(ptx::bf16hi_to_f32(wv[e]), kLog2e, bias[2 * e + 1]);
                        }
                    }
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float u = fmaf(__uint_as_float(s[cc * 8 + e]), p.scale_log2, bias[e]);
                        s[cc * 8 + e] = __float_as_uint(u);
                        rmax = fmaxf(rmax, u);
                    }
                }
                __syncwarp();
                if (lane == 0) {
                    ptx::mbar_arrive(bar(C::BAR_ME + w * C::M_STAGES + mstage));
                    if (HAS_PAIR) ptx::mbar_arrive(bar(C::BAR_BE + bstage));
                }

                const float m_new = fmaxf(m_used, rmax);
                const bool rescale = m_new > m_used + kRescaleThreshold;
                float alpha = 1.f;
                if (rescale) {
                    alpha = ptx::ex2_approx(m_used - m_new);  // 0 while m_used is -inf
                    m_used = m_new;
                }
                const float m_safe = (m_used == -INFINITY) ? 0.f : m_used;
                float rsum = 0.f;
                uint32_t pk[64];
#pragma unroll
                for (int c = 0; c < 64; ++c) {
                    const float p0 = ptx::ex2_approx(__uint_as_float(s[2 * c]) - m_safe);
                    const float p1 = ptx::ex2_approx(__uint_as_float(s[2 * c + 1]) - m_safe);
                    rsum += p0 + p1;
                    pk[c] = ptx::pack_bf16x2(p0, p1);
                }
                l = l * alpha + rsum;

                if (j > 0) {
                    // P and O of the previous block are in use until its P.V is done.
                    ok = wait_warp(bar(C::BAR_PE + w), (j - 1) & 1, abort_flag);
                    if (!ok) break;
                    ptx::tc_fence_after();
                    if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
                        for (int dc = 0; dc < D; dc += 16) {
                            uint32_t o[16];
                            ptx::tmem_ld_x16(tO + dc, o);
                            ptx::tmem_ld_wait_x16(o);
#pragma unroll
                            for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                            ptx::tmem_st_x16(tO + dc, o);
                        }
                    }
                }
                ptx::tmem_st_x32(tP, pk);
                ptx::tmem_st_x32(tP + 32, pk + 32);
                ptx::tmem_st_wait();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(bar(C::BAR_PF + w));
            }
            // ---------------------------------------------------------- epilogue
            if (ok) ok = wait_warp(bar(C::BAR_PE + w), (nkb - 1) & 1, abort_flag);
            if (ok) {
                ptx::tc_fence_after();
                const int n = n0 + w;
                const int row = q0 + r;
                const float inv_l = l > 0.f ? 1.f / l : 0.f;
                uint16_t* orow = p.out + ((size_t(b) * p.N + n) * size_t(p.S) + size_t(row)) * size_t(p.H) * D +
                                 size_t(h) * D;
#pragma unroll
                for (int dc = 0; dc < D; dc += 16) {
                    uint32_t o[16];
                    ptx::tmem_ld_x16(tO + dc, o);
                    ptx::tmem_ld_wait_x16(o);
                    uint32_t packed[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        packed[e] = ptx::pack_bf16x2(__uint_as_float(o[2 * e]) * inv_l,
                                                     __uint_as_float(o[2 * e + 1]) * inv_l);
                    if (row < p.S) {
                        uint4* dst = reinterpret_cast<uint4*>(orow + dc);
                        dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
                        dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
                    }
                }
                if (row < p.S) {
                    const float lse = l > 0.f ? (m_used + ptx::lg2_approx(l)) * kLn2 + csub_s[w] : -INFINITY;
                    p.lse[((size_t(b) * p.N + n) * p.H + h) * size_t(p.S) + row] = lse;
                }
            }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace evo
