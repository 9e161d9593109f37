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
//    softmax warpgroups.  CTAs are numbered query block fastest, then head,
//    so the CTAs that share one (n, h) K/V slice, and the four heads that
//    share each 256 B stretch of a Q/K/V row, run at the same time and hit L2.
//  * Warp roles (608 threads, 19 warps): warp 0 issues TMA loads (Q once; K,
//    V and bias tiles through rings of mbarrier-tracked stages); warp 1 issues
//    tcgen05 MMAs from one thread; warp 2 turns the mask row into a
//    log2-scaled fp32 vector per key block (with the per-(b,n) rebase below);
//    warps 3-18 are softmax warps, eight per slice, each owning 16 query rows
//    (TMEM lanes) through the 16-lane `16x64b` tensor-memory shape: the two
//    threads of a row hold its even and its odd key columns, so a row maximum
//    is one shuffle and no barrier couples the softmax warps; they drift apart
//    and the exp unit of one overlaps the FMA/ALU work of another.  Each
//    softmax warp also converts 16 rows of its slice's V tile to fp16 before
//    it reports P ready, so the P.V MMA that waits for P also finds V
//    converted.
//  * Tensor memory (512 columns): one S = Q K^T buffer (128 fp32 columns)
//    that the two slices take turns in, two P buffers per slice (softmax
//    numerators as fp16, 64 columns each) and one O accumulator per slice.
//    A slice's next Q K^T is issued as soon as the other slice has pulled its
//    S into registers, which staggers the two slices by about half a block;
//    with two P buffers a softmax warp writes block j+1's P while block j's
//    P.V is still running, so no warp waits for the tensor core in the steady
//    state (only a rare O rescale waits for the previous P.V).
//  * P is packed from a thread's own (interleaved) columns, so within every
//    group of four keys the MMA sees key order 0, 2, 1, 3; the V conversion
//    swaps rows 1 and 2 of every group of four to match (a permutation of
//    the contraction index leaves P.V unchanged).
//  * P is rounded to fp16, not bf16: its 11-bit significand keeps the P.V
//    rounding error eight times below bf16's, which holds |dO| under 1e-2
//    next to the bf16 rounding of O itself.  MMA operands share one type, so
//    V is converted to fp16 in shared memory (exact for |V| <= 65504; larger
//    values are reported as EVO_ERR_RANGE).
//  * For D <= 32 the row sum comes from the tensor core: each V stage is
//    followed by a constant tile whose first column is 1.0, and the P.V MMA
//    runs with N = D + 16, so O's column D accumulates sum_j P_j (the same
//    rounded P that weights V) and is rescaled together with O.
//  * Online softmax in base 2: u = s*log2(e)/sqrt(D) + (pair + mask - c)*log2(e),
//    p = 2^(u - m), with packed f32x2 FMA/ADD.  The running maximum m is only
//    moved when the block maximum exceeds it by more than 8 (p <= 256, exact
//    after the final division by the row sum); moving it rescales O in
//    tensor memory.
//  * Mask rebase: the mask warp keeps c = the largest mask value seen so far
//    for each slice (an online max over key blocks), hands the softmax
//    (mask - c) * log2(e), and publishes c with every block; when c grows the
//    softmax lowers its running max by the same amount, and the final c is
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
    int num_qb;            // query blocks of 128
    int num_np;            // n pairs, ceil(N / 2)
    float scale_log2;      // log2(e) / sqrt(D)
};

constexpr int kBM = 128;          // query rows per slice tile
constexpr int kBN = 128;          // keys per block
constexpr int kThreads = 608;          // 3 helper warps + 16 softmax warps (104 registers each)
constexpr int kFirstSoftmaxWarp = 3;
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
    static constexpr bool SUM_MMA = D <= 32;          // row sum from a ones column of V
    static constexpr int OW = D + (SUM_MMA ? 16 : 0); // O accumulator columns
    static constexpr int K_STAGES = (D <= 32) ? 4 : 3;
    static constexpr int V_STAGES = (D <= 32) ? 4 : 3;
    static constexpr int V_STRIDE = SUM_MMA ? 2 * TILE : TILE;  // V tile (+ ones tile)
    static constexpr int M_STAGES = 2;
    static constexpr int BIAS_BYTES = kBM * kBN * 2;  // two 128x64 boxes, 128 B swizzle
    static constexpr int B_STAGES = HAS_PAIR ? 2 : 0;
    // shared-memory map (offsets from a 1024-aligned base)
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + 2 * TILE;
    static constexpr int OFF_V = OFF_K + K_STAGES * TILE;
    static constexpr int OFF_BIAS = OFF_V + V_STAGES * V_STRIDE;
    static constexpr int OFF_MASK = OFF_BIAS + B_STAGES * BIAS_BYTES;  // [2][M_STAGES][128] f32
    static constexpr int OFF_MC = OFF_MASK + 2 * M_STAGES * kBN * 4;  // [2][M_STAGES] f32 rebase c
    static constexpr int OFF_BAR = OFF_MC + 64;
    // barrier indices
    static constexpr int BAR_Q = 0;
    static constexpr int BAR_KF = 1;
    static constexpr int BAR_KE = BAR_KF + K_STAGES;
    static constexpr int BAR_VF = BAR_KE + K_STAGES;   // V landed (bf16)
    static constexpr int BAR_VE = BAR_VF + V_STAGES;
    static constexpr int BAR_BF = BAR_VE + V_STAGES;
    static constexpr int BAR_BE = BAR_BF + 2;
    static constexpr int BAR_MF = BAR_BE + 2;           // [2][M_STAGES]
    static constexpr int BAR_ME = BAR_MF + 2 * M_STAGES;
    static constexpr int BAR_SF = BAR_ME + 2 * M_STAGES;  // [2] S of slice w ready
    static constexpr int BAR_SE = BAR_SF + 2;             // [2] slice w has read S
    // P ready / P.V done, one barrier per P buffer: a slice can be one block
    // ahead of the MMA issuer, and block j and j + 1 use different barriers,
    // so a wait on block j's phase never sees block j + 2's.
    static constexpr int BAR_PF = BAR_SE + 2;             // [2 slices][2 buffers] P written, V converted
    static constexpr int BAR_PE = BAR_PF + 4;             // [2 slices][2 buffers] P.V done
    static constexpr int BAR_DRAIN = BAR_PE + 4;
    static constexpr int NUM_BARS = BAR_DRAIN + 1;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;  // tmem slot, abort flag
    static constexpr int USED = OFF_MISC + 16;
    // Request at least 116 KB so that two CTAs never share an SM: each CTA
    // allocates all 512 tensor-memory columns.
    static constexpr int SMEM_BYTES = (USED + 1024 > 116 * 1024) ? USED + 1024 : 116 * 1024;
    static_assert(USED + 1024 <= 227 * 1024, "shared memory");
    // tensor-memory columns
    static constexpr uint32_t TM_S = 0;     // shared by both slices
    static constexpr uint32_t TM_P0 = 128;  // + 64 * (2 * w + buffer)
    static constexpr uint32_t TM_O0 = 384;  // + OW * w
    static constexpr uint32_t TMEM_COLS = 512;
    static_assert(TM_O0 + 2 * OW <= TMEM_COLS, "tensor memory");
    // instruction descriptors, fp32 accumulate, M = 128:
    // Q K^T: bf16 x bf16, both K-major, N = 128 keys
    static constexpr uint32_t IDESC_QK =
        (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t(kBN) >> 3) << 17) | ((uint32_t(kBM) >> 4) << 24);
    // P V: fp16 x fp16, P from tensor memory, V MN-major, N = OW
    static constexpr uint32_t IDESC_PV =
        (1u << 4) | (0u << 7) | (0u << 10) | (1u << 16) | ((uint32_t(OW) >> 3) << 17) | ((uint32_t(kBM) >> 4) << 24);
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

// Converts 16 rows (keys) of a TMA-swizzled bf16 V tile to fp16 in place and
// swaps rows 4g+1 and 4g+2 of every group of four (the key order in which the
// softmax packs P).  Row r's 16-byte chunk c sits at chunk c ^ ((r * ROW /
// 128) % (ROW / 16)) of the row.  A value beyond the fp16 range becomes
// +-inf and surfaces as a non-finite row sum or output, which the epilogue
// reports as EVO_ERR_RANGE.
// The 16 B chunks of V a softmax warp converts: rows row0 .. row0+15 of the
// tile, spread over the lanes.  Offsets are computed once per thread.
template <int ROW>
struct VConvPlan {
    static constexpr int CHUNKS = ROW / 16;            // 16 B chunks per row
    static constexpr int ITEMS = 16 * CHUNKS;          // 16 rows x CHUNKS
    static constexpr int PER_LANE = (ITEMS + 31) / 32;
    uint32_t src[PER_LANE], dst[PER_LANE];
    __device__ __forceinline__ static uint32_t at(int r, int c) {
        const int sw = ((r * ROW) >> 7) & (CHUNKS - 1);  // row r's chunk c sits at chunk c ^ sw
        return uint32_t(r * ROW) + uint32_t((c ^ sw) << 4);
    }
    __device__ __forceinline__ VConvPlan(int row0, int lane) {
#pragma unroll
        for (int k = 0; k < PER_LANE; ++k) {
            const int item = (lane + 32 * k) % ITEMS;  // lanes past the end redo an item (same result)
            const int rr = item / CHUNKS, c = item % CHUNKS;
            const int swapped = (rr & ~3) | ((rr & 1) << 1) | ((rr >> 1) & 1);  // rows 1 and 2 of each 4
            src[k] = at(row0 + rr, c);
            dst[k] = at(row0 + swapped, c);
        }
    }
    // Converts bf16 -> fp16 in place with the row swap.  Every lane reads all its
    // chunks before any lane writes.
    __device__ __forceinline__ void run(uint32_t tile) const {
        uint4 v[PER_LANE];
#pragma unroll
        for (int k = 0; k < PER_LANE; ++k) v[k] = ptx::ld_shared_v4(tile + src[k]);
        __syncwarp();
#pragma unroll
        for (int k = 0; k < PER_LANE; ++k) {
            uint32_t o[4];
            const uint32_t wv[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) o[e] = ptx::pack_f16x2(ptx::bf16lo_to_f32(wv[e]), ptx::bf16hi_to_f32(wv[e]));
            ptx::st_shared_v4(tile + dst[k], make_uint4(o[0], o[1], o[2], o[3]));
        }
    }
};

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
    // CTA index: query block fastest, then head, then n pair, then batch
    int rest = blockIdx.x;
    const int qb = rest % p.num_qb;
    rest /= p.num_qb;
    const int h = rest % p.H;
    rest /= p.H;
    const int np = rest % p.num_np;
    const int b = rest / p.num_np;
    const int n0 = np * 2;
    const int q0 = qb * kBM;
    const int bh = b * p.H + h;
    const int n_valid = (p.N - n0) < 2 ? (p.N - n0) : 2;
    const int nkb = p.num_kb;

    auto bar = [&](int i) -> uint32_t { return sb + C::OFF_BAR + 8u * uint32_t(i); };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
    float* mc_s = reinterpret_cast<float*>(smem + C::OFF_MC);  // [w * M_STAGES + stage]

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
            ptx::mbar_init(bar(C::BAR_BE + s), 8 * n_valid);
        }
        for (int s = 0; s < 2 * C::M_STAGES; ++s) {
            ptx::mbar_init(bar(C::BAR_MF + s), 32);
            ptx::mbar_init(bar(C::BAR_ME + s), 8);
        }
        for (int w = 0; w < 2; ++w) {
            ptx::mbar_init(bar(C::BAR_SF + w), 1);
            ptx::mbar_init(bar(C::BAR_SE + w), 8);
            ptx::mbar_init(bar(C::BAR_PF + 2 * w), 8);
            ptx::mbar_init(bar(C::BAR_PF + 2 * w + 1), 8);
            ptx::mbar_init(bar(C::BAR_PE + 2 * w), 1);
            ptx::mbar_init(bar(C::BAR_PE + 2 * w + 1), 1);
        }
        ptx::mbar_init(bar(C::BAR_DRAIN), 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (C::SUM_MMA && warp == 2) {
        // Constant tiles after each V stage: column 0 = 1.0 (fp16), rest 0,
        // laid out with the same swizzle as V (16 B chunk c of row r sits at
        // chunk c ^ ((r * ROW / 128) % (ROW / 16))).
        for (int s = 0; s < C::V_STAGES; ++s) {
            const uint32_t base = sb + C::OFF_V + uint32_t(s * C::V_STRIDE + C::TILE);
            for (int c = lane; c < C::TILE / 16; c += 32)
                ptx::st_shared_v4(base + uint32_t(c) * 16u, make_uint4(0u, 0u, 0u, 0u));
        }
        __syncwarp();
        for (int s = 0; s < C::V_STAGES; ++s) {
            const uint32_t base = sb + C::OFF_V + uint32_t(s * C::V_STRIDE + C::TILE);
            for (int r = lane; r < kBM; r += 32) {
                const uint32_t chunk = uint32_t((r * C::ROW) >> 7) & uint32_t(C::ROW / 16 - 1);
                asm volatile("st.shared.u16 [%0], %1;" ::"r"(base + uint32_t(r * C::ROW) + chunk * 16u),
                             "h"(uint16_t(0x3C00)) : "memory");
            }
        }
        ptx::fence_proxy_async_smem();
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
                    ptx::tma_load_4d(sb + C::OFF_V + s * C::V_STRIDE, &tm_v, bar(C::BAR_VF + s), 0, h, j * kBN,
                                     bn0 + w);
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
                if (!wait_fast(bar(C::BAR_KF + s), (k_used / C::K_STAGES) & 1, abort_flag)) return false;
                ptx::tc_fence_after();
                const uint64_t a = desc_k_major<C::ROW>(sb + C::OFF_Q + w * C::TILE);
                const uint64_t bdesc = desc_k_major<C::ROW>(sb + C::OFF_K + s * C::TILE);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)  // 16 bf16 = 32 B per K step
                    ptx::mma_ss(tmem + C::TM_S, a + uint64_t(2 * kk), bdesc + uint64_t(2 * kk),
                                C::IDESC_QK, kk > 0 ? 1u : 0u);
                ptx::mma_commit(bar(C::BAR_KE + s));
                ptx::mma_commit(bar(C::BAR_SF + w));
                ++k_used;
                return true;
            };
            auto issue_pv = [&](int w, int j) -> bool {
                const int s = v_used % C::V_STAGES;
                // P of block j written and V converted (buffer j & 1, its (j >> 1)-th use)
                if (!wait_fast(bar(C::BAR_PF + 2 * w + (j & 1)), (j >> 1) & 1, abort_flag)) return false;
                ptx::tc_fence_after();
                const uint64_t bdesc = desc_mn_major<C::ROW>(sb + C::OFF_V + s * C::V_STRIDE, C::TILE);
                const uint32_t a_tmem = tmem + C::TM_P0 + 64u * uint32_t(2 * w + (j & 1));
#pragma unroll
                for (int kk = 0; kk < kBN / 16; ++kk)  // 16 keys per K step = 16 rows of V
                    ptx::mma_ts(tmem + C::TM_O0 + uint32_t(C::OW) * w, a_tmem + 8u * kk,
                                bdesc + uint64_t((16 * C::ROW * kk) >> 4), C::IDESC_PV, (j > 0 || kk > 0) ? 1u : 0u);
                ptx::mma_commit(bar(C::BAR_VE + s));
                ptx::mma_commit(bar(C::BAR_PE + 2 * w + (j & 1)));
                ++v_used;
                return true;
            };
            // The S buffer is shared: slice 0's Q K^T for block j follows the last
            // slice's read of block j-1, slice 1's follows slice 0's read of block j.
            for (int j = 0; j < nkb && ok; ++j) {
                if (j > 0) ok = wait_fast(bar(C::BAR_SE + (n_valid - 1)), (j - 1) & 1, abort_flag);
                ok = ok && issue_qk(0);
                if (n_valid == 2) ok = ok && wait_fast(bar(C::BAR_SE + 0), j & 1, abort_flag) && issue_qk(1);
                if (j > 0)
                    for (int w = 0; w < n_valid && ok; ++w) ok = issue_pv(w, j - 1);
            }
            for (int w = 0; w < n_valid && ok; ++w) ok = issue_pv(w, nkb - 1);
            if (!ok) {
                // Wait for every MMA this thread issued before tensor memory is freed.
                ptx::mma_commit(bar(C::BAR_DRAIN));
                wait_bounded(bar(C::BAR_DRAIN), 0, nullptr);
            }
        }
        __syncwarp();
    } else if (warp == 2) {
        // ------------------------------------------------------------ mask warp
        // Lane l handles keys l, l+32, l+64, l+96 of each block, for both slices;
        // the next block's raw values are fetched while this block is processed.
        // With a pair bias it also waits for the block's bias tile before
        // releasing the stage, so one barrier tells a softmax warp both are ready.
        const uint16_t* mrow[2] = {nullptr, nullptr};
        for (int w = 0; w < n_valid; ++w)
            if (p.mask != nullptr) mrow[w] = p.mask + (size_t(b) * p.N + n0 + w) * size_t(p.S);
        float c_run[2] = {-INFINITY, -INFINITY};
        uint32_t raw[2][4];
        auto fetch = [&](int j) {
#pragma unroll
            for (int w = 0; w < 2; ++w)
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int key = j * kBN + lane + 32 * k;
                    raw[w][k] = (mrow[w] != nullptr && key < p.S) ? uint32_t(mrow[w][key]) : 0u;
                }
        };
        fetch(0);
        bool ok = true;
        for (int j = 0; j < nkb && ok; ++j) {
            uint32_t cur[2][4];
#pragma unroll
            for (int w = 0; w < 2; ++w)
#pragma unroll
                for (int k = 0; k < 4; ++k) cur[w][k] = raw[w][k];
            if (j + 1 < nkb) fetch(j + 1);
            const int stage = j % C::M_STAGES;
            const uint32_t ph = (j / C::M_STAGES) & 1;
            if (HAS_PAIR && !wait_warp(bar(C::BAR_BF + (j & 1)), (j >> 1) & 1, abort_flag)) { ok = false; break; }
            for (int w = 0; w < n_valid && ok; ++w) {
                float v[4];
                float bmax = -INFINITY;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int key = j * kBN + lane + 32 * k;
                    v[k] = key < p.S ? __uint_as_float(cur[w][k] << 16) : -INFINITY;  // absent mask: 0
                    bmax = fmaxf(bmax, v[k]);
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, o));
                c_run[w] = fmaxf(c_run[w], bmax);
                const float csub = (c_run[w] == -INFINITY) ? 0.f : c_run[w];  // all -inf so far: keep -inf logits
                if (!wait_warp(bar(C::BAR_ME + w * C::M_STAGES + stage), ph ^ 1, abort_flag)) { ok = false; break; }
                // even keys first, then odd keys: a softmax thread reads its own parity
                float* dst = reinterpret_cast<float*>(smem + C::OFF_MASK) + (w * C::M_STAGES + stage) * kBN;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int t = lane + 32 * k;
                    dst[(t & 1) * (kBN / 2) + (t >> 1)] = (v[k] - csub) * kLog2e;
                }
                if (lane == 0) mc_s[w * C::M_STAGES + stage] = csub;
                ptx::mbar_arrive(bar(C::BAR_MF + w * C::M_STAGES + stage));
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax
        const int sidx = warp - kFirstSoftmaxWarp;  // 0..15
        const int w = sidx >> 3;                    // slice (n0 + w)
        const int quarter = warp & 3;               // this warp may touch TMEM lanes 32*quarter .. +31
        const int sub = (sidx >> 2) & 1;            // which 16 of those 32 lanes
        const int lane0 = quarter * 32 + sub * 16;  // first row of the warp
        const int par = (lane >> 1) & 1;            // key parity this thread holds
        const int r = lane0 + (lane >> 2) + 8 * (lane & 1);  // query row in the tile == TMEM lane
        if (w < n_valid) {
            const uint32_t lane_base = uint32_t(lane0) << 16;
            const uint32_t tS = tmem + lane_base + C::TM_S;
            const uint32_t tP0 = tmem + lane_base + C::TM_P0 + 128u * w;  // + 64 * buffer
            const uint32_t tO = tmem + lane_base + C::TM_O0 + uint32_t(C::OW) * w;
            const float2 l2e2 = make_float2(kLog2e, kLog2e);
            const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
            const float2 one2 = make_float2(1.f, 1.f);
            // byte selector that moves this thread's bf16 half of a word into the high half of a float
            const uint32_t psel = par ? 0x3244u : 0x1044u;
            const VConvPlan<C::ROW> vplan(16 * (sidx & 7), lane);
            float m_used = -INFINITY;
            float c_cur = 0.f;  // mask rebase the current m_used and P are relative to
            float l = 0.f;      // this thread's share of the row sum when the tensor core does not keep it
            bool ok = true;
            for (int j = 0; j < nkb; ++j) {
                // s[i] = S[r][2i + par], i = 0..63
                uint32_t s[64];
                ok = wait_warp(bar(C::BAR_SF + w), j & 1, abort_flag);
                if (!ok) break;
                ptx::tc_fence_after();
                ptx::tmem_ld_16x64b_x64_wait(tS, s);
                ptx::tc_fence_before();
                ptx::mbar_arrive_elect(bar(C::BAR_SE + w));

                // mask vector (and, with a pair bias, the bias tile: the mask warp waited for it)
                const int mstage = j % C::M_STAGES;
                ok = wait_warp(bar(C::BAR_MF + w * C::M_STAGES + mstage), (j / C::M_STAGES) & 1, abort_flag);
                if (!ok) break;
                const int bstage = j & 1;
                {
                    // the mask rebase grew: earlier logits are relative to a smaller c
                    const float cs = mc_s[w * C::M_STAGES + mstage];
                    if (cs != c_cur) {
                        m_used -= (cs - c_cur) * kLog2e;
                        c_cur = cs;
                    }
                }
                const uint32_t maddr = sb + C::OFF_MASK + uint32_t((w * C::M_STAGES + mstage) * kBN * 4) +
                                       uint32_t(par * (kBN / 2) * 4);
                // row r starts 128 B-aligned, so chunk k of it sits at (row start | (r % 8) << 4) ^ (k << 4)
                const uint32_t brow = (sb + C::OFF_BIAS + uint32_t(bstage * C::BIAS_BYTES) + uint32_t(r * 128)) |
                                      uint32_t((r & 7) << 4);
                float rmax0 = -INFINITY, rmax1 = -INFINITY;
#pragma unroll
                for (int c = 0; c < 16; ++c) {  // bias chunk c: keys 8c .. 8c+7, this thread's 4 of them
                    const float4 mv = ptx::ld_shared_f4(maddr + c * 16);
                    float2 t0 = make_float2(mv.x, mv.y), t1 = make_float2(mv.z, mv.w);
                    if (HAS_PAIR) {
                        // 128 B swizzle: chunk (c % 8) of row r in box c / 8 sits at chunk (c % 8) ^ (r % 8)
                        const uint4 pw =
                            ptx::ld_shared_v4((brow ^ uint32_t((c & 7) << 4)) + uint32_t((c >> 3) * (C::BIAS_BYTES / 2)));
                        const float b0 = __uint_as_float(__byte_perm(pw.x, 0u, psel));
                        const float b1 = __uint_as_float(__byte_perm(pw.y, 0u, psel));
                        const float b2 = __uint_as_float(__byte_perm(pw.z, 0u, psel));
                        const float b3 = __uint_as_float(__byte_perm(pw.w, 0u, psel));
                        t0 = __ffma2_rn(make_float2(b0, b1), l2e2, t0);
                        t1 = __ffma2_rn(make_float2(b2, b3), l2e2, t1);
                    }
                    const int k = 4 * c;
                    const float2 u0 = __ffma2_rn(make_float2(__uint_as_float(s[k]), __uint_as_float(s[k + 1])), sc2, t0);
                    const float2 u1 =
                        __ffma2_rn(make_float2(__uint_as_float(s[k + 2]), __uint_as_float(s[k + 3])), sc2, t1);
                    s[k] = __float_as_uint(u0.x);
                    s[k + 1] = __float_as_uint(u0.y);
                    s[k + 2] = __float_as_uint(u1.x);
                    s[k + 3] = __float_as_uint(u1.y);
                    rmax0 = max3f(rmax0, u0.x, u0.y);
                    rmax1 = max3f(rmax1, u1.x, u1.y);
                }
                ptx::mbar_arrive_elect(bar(C::BAR_ME + w * C::M_STAGES + mstage));
                if (HAS_PAIR) ptx::mbar_arrive_elect(bar(C::BAR_BE + bstage));
                float rmax = fmaxf(rmax0, rmax1);
                rmax = fmaxf(rmax, __shfl_xor_sync(0xffffffffu, rmax, 2));  // the other parity of the row

                const float m_new = fmaxf(m_used, rmax);
                const bool rescale = m_new > m_used + kRescaleThreshold;
                float alpha = 1.f;
                if (rescale) {
                    alpha = ptx::ex2_approx(m_used - m_new);  // 0 while m_used is -inf
                    m_used = m_new;
                }
                const float m_safe = (m_used == -INFINITY) ? 0.f : m_used;
                const float2 nm2 = make_float2(-m_safe, -m_safe);

                float2 acc = make_float2(0.f, 0.f);
                // register i of a store lands in P column 2i + par: it packs this thread's keys
                // 2(2i') + par and 2(2i'+1) + par (MMA key order 0, 2, 1, 3)
                uint32_t pk[32];
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const float2 x =
                        __ffma2_rn(make_float2(__uint_as_float(s[2 * c]), __uint_as_float(s[2 * c + 1])), one2, nm2);
                    const float p0 = ptx::ex2_approx(x.x);
                    const float p1 = ptx::ex2_approx(x.y);
                    if (!C::SUM_MMA) acc = __ffma2_rn(make_float2(p0, p1), one2, acc);
                    pk[c] = ptx::pack_f16x2(p0, p1);
                }
                if (!C::SUM_MMA) l = l * alpha + (acc.x + acc.y);

                // P buffer j & 1 was last read by the P.V of block j - 2
                const uint32_t tP = tP0 + 64u * uint32_t(j & 1);
                if (j >= 2) {
                    ok = wait_warp(bar(C::BAR_PE + 2 * w + (j & 1)), ((j - 2) >> 1) & 1, abort_flag);
                    if (!ok) break;
                    ptx::tc_fence_after();
                }
                if (j > 0 && __any_sync(0xffffffffu, rescale)) {
                    // O holds every block before j once the P.V of block j - 1 is done
                    ok = wait_warp(bar(C::BAR_PE + 2 * w + ((j - 1) & 1)), ((j - 1) >> 1) & 1, abort_flag);
                    if (!ok) break;
                    ptx::tc_fence_after();
                    {
#pragma unroll
                        for (int dc = 0; dc < C::OW; dc += 16) {  // 8 repeats of 2 columns
                            uint32_t o[8];
                            ptx::tmem_ld_16x64b_x8(tO + dc, o);
                            ptx::tmem_ld_wait_x8(o);
#pragma unroll
                            for (int e = 0; e < 8; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                            ptx::tmem_st_16x64b_x8(tO + dc, o);
                        }
                    }
                }
                ptx::tmem_st_16x64b_x16(tP, pk);
                ptx::tmem_st_16x64b_x16(tP + 32, pk + 16);

                // this warp's 16 rows of V_j for slice w: bf16 -> fp16 in place, key order 0,2,1,3
                {
                    const int vi = j * n_valid + w;  // index of the tile in the producer's V order
                    const int vs = vi % C::V_STAGES;
                    ok = wait_warp(bar(C::BAR_VF + vs), (vi / C::V_STAGES) & 1, abort_flag);
                    if (!ok) break;
                    vplan.run(sb + C::OFF_V + uint32_t(vs * C::V_STRIDE));
                    ptx::fence_proxy_async_smem();  // generic-proxy writes -> tensor-core reads
                }
                ptx::tmem_st_wait();
                ptx::tc_fence_before();
                ptx::mbar_arrive_elect(bar(C::BAR_PF + 2 * w + (j & 1)));
            }
            // ---------------------------------------------------------- epilogue
            if (ok) ok = wait_warp(bar(C::BAR_PE + 2 * w + ((nkb - 1) & 1)), ((nkb - 1) >> 1) & 1, abort_flag);
            if (ok) {
                ptx::tc_fence_after();
                const int n = n0 + w;
                const int row = q0 + r;
                if (C::SUM_MMA) {
                    uint32_t o[8];
                    ptx::tmem_ld_16x64b_x8(tO + D, o);  // column D (even) holds the row sum
                    ptx::tmem_ld_wait_x8(o);
                    l = __uint_as_float(o[0]);
                    l = __shfl_sync(0xffffffffu, l, lane & ~2);  // from the even-column thread
                } else {
                    l += __shfl_xor_sync(0xffffffffu, l, 2);
                }
                const float inv_l = l > 0.f ? 1.f / l : 0.f;
                // thread (row, par) holds d = 2i + par; swap halves with the partner so that
                // par 0 stores d in [0, D/2) and par 1 stores d in [D/2, D)
                constexpr int NV = D / 2;  // values per thread
                uint32_t o[NV];
#pragma unroll
                for (int dc = 0; dc < D; dc += 16) {
                    ptx::tmem_ld_16x64b_x8(tO + dc, o + dc / 2);
                }
                ptx::tmem_ld_wait_x8(o);
#pragma unroll
                for (int i = 8; i < NV; i += 8) ptx::reg_fence_x8(o + i);
                bool finite = (l < INFINITY);  // an fp16 overflow of V shows up here or in O
                // value i holds d = 2i + par.  par 0 stores d in [0, NV): its own even d and the
                // partner's odd d of slots 0..NV/2-1; par 1 stores d in [NV, D) from slots NV/2..NV-1.
                float mine[NV];
#pragma unroll
                for (int k = 0; k < NV / 2; ++k) {
                    const float lo = __uint_as_float(o[k]) * inv_l;           // d = 2k + par
                    const float hi = __uint_as_float(o[k + NV / 2]) * inv_l;  // d = 2k + NV + par
                    finite = finite && fabsf(lo) < INFINITY && fabsf(hi) < INFINITY;
                    const float recv = __shfl_xor_sync(0xffffffffu, par ? lo : hi, 2);
                    mine[2 * k] = par ? recv : lo;
                    mine[2 * k + 1] = par ? hi : recv;
                }
                if (row < p.S) {
                    uint16_t* orow = p.out + ((size_t(b) * p.N + n) * size_t(p.S) + size_t(row)) * size_t(p.H) * D +
                                     size_t(h) * D + size_t(NV * par);
#pragma unroll
                    for (int k = 0; k < NV; k += 8) {
                        uint4 v;
                        v.x = ptx::pack_bf16x2(mine[k + 0], mine[k + 1]);
                        v.y = ptx::pack_bf16x2(mine[k + 2], mine[k + 3]);
                        v.z = ptx::pack_bf16x2(mine[k + 4], mine[k + 5]);
                        v.w = ptx::pack_bf16x2(mine[k + 6], mine[k + 7]);
                        *reinterpret_cast<uint4*>(orow + k) = v;
                    }
                    if (!finite) record_status(EVO_ERR_RANGE);
                    if (par == 0) {
                        const float lse = l > 0.f ? (m_used + ptx::lg2_approx(l)) * kLn2 + c_cur : -INFINITY;
                        p.lse[((size_t(b) * p.N + n) * p.H + h) * size_t(p.S) + row] = lse;
                    }
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
