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
//  * Warp roles (384 threads, 12 warps): warp 0 issues TMA loads (Q once; K
//    and bias tiles through rings of mbarrier-tracked stages); warps 1 and 2
//    serve slice 0 and 1: each loads its slice's V tiles (a ring of its own),
//    turns the mask row into the mask columns of the score MMA (below) and
//    issues the slice's tcgen05 MMAs from one thread, in a fixed order that
//    follows the softmax, each step a blocking wait on one barrier; warp 3
//    converts the V tiles of both slices to fp16, so that no MMA issue waits
//    behind a V load or its conversion (for D = 64, whose tiles are twice as
//    large, each helper converts the first half of its own); warps 4-7 and
//    8-11 are the softmax
//    warpgroups of slice 0 and 1 (warp w reaches tensor-memory lanes
//    32 * (w % 4) ..).  setmaxnreg moves registers from the first warpgroup
//    to the softmax warpgroups.  A softmax thread
//    owns one query row (one tensor-memory lane) and all 128 keys of a block,
//    so the row maximum needs no shuffle and the bias row is read with 16 B
//    loads it uses in full.
//  * Tensor memory (512 columns): per slice one S = Q K^T buffer (128 fp32
//    columns), one P buffer (softmax numerators as fp16, 64 columns) and one
//    O accumulator.  A slice's next Q K^T is issued as soon as its softmax has
//    pulled S into registers, so S(j+1) is computed while the softmax works on
//    block j, and P(j) is only overwritten after P(j).V has finished.
//  * The mask bias enters through the tensor core: the score MMA gets one more
//    K=16 step whose A tile holds 1, 1, 1 in columns 0-2 of every query row and
//    whose B tile holds, for key j, three bf16 numbers hi + mid + lo that sum
//    exactly to the fp32 value (mask[j] - c) * sqrt(D) (c: rebase, below).  S
//    then already includes the mask term, so the softmax adds only the pair
//    bias.  Keys beyond S get -inf there.
//  * P is rounded to fp16, not bf16: its 11-bit significand keeps the P.V
//    rounding error eight times below bf16's, which holds |dO| under 1e-2
//    next to the bf16 rounding of O itself.  MMA operands share one type, so
//    V is converted to fp16 in shared memory (exact for |V| <= 65504; larger
//    values are reported as EVO_ERR_RANGE).
//  * For D <= 32 the row sum comes from the tensor core: the P.V MMA runs
//    with N = D + 16 over V followed (through the descriptor's atom stride) by
//    one constant tile whose first column is 1.0, so O's column D accumulates
//    sum_j P_j (the same rounded P that weights V) and is rescaled with O.
//  * Online softmax in base 2: with t = S + pair * sqrt(D) (fp32, packed
//    f32x2 FMA), p = 2^(t * log2(e) / sqrt(D) - m).  The running maximum m is
//    only moved when the block maximum exceeds it by more than 12 (p <= 4096,
//    far inside the fp16 range, and exact after the final division by the row
//    sum); moving it rescales O in tensor memory.
//  * Mask rebase: the slice's helper warp keeps c = the largest mask value
//    seen so far (an online max over key blocks) and subtracts it before the
//    mask enters the MMA; when c grows the softmax lowers its running max by
//    the same amount, and the final c is added back to the LSE.  The guide
//    builds masks as 1e9*(mask-1) (section 5.2); for an n whose every key is
//    masked that is a constant shift of the row, and the rebase keeps fp32
//    from rounding every logit to -1e9.
//  * Every wait is bounded (about two seconds); on expiry the CTA records
//    EVO_ERR_TIMEOUT, drains its own in-flight copies and MMAs, frees tensor
//    memory and exits.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
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
    int aug;               // mask columns in the score MMA (a mask, or a ragged last key block)
    float scale_log2;      // log2(e) / sqrt(D)
    float sqrt_d;          // sqrt(D)
};

constexpr int kBM = 128;          // query rows per slice tile
constexpr int kBN = 128;          // keys per block
constexpr int kThreads = 384;     // helper warpgroup (producer, 2 slice helpers, V converter) + 2 softmax warpgroups
constexpr int kFirstSoftmaxWarp = 4;
// Register split (setmaxnreg): the helper warpgroup hands registers to the two
// softmax warpgroups, which keep a block's 128 scores in registers and need
// room beside them to overlap independent work.  The split must not exceed
// the 384 x 168 registers the block is launched with.
constexpr int kHelperRegs = 96;
constexpr int kSoftmaxRegs = 200;
static_assert(128 * kHelperRegs + 256 * kSoftmaxRegs <= 384 * 168, "register split");
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 12.0f;  // log2 units: p <= 2^12 (fp16 P) between rescales
// Masks more than this far below a row's running mask maximum (natural-log
// units) are treated as -inf; see the mask-column writers.
constexpr float kMaskFloor = 16384.0f;


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
    static constexpr int K_STAGES = (D <= 32) ? 4 : 2;  // K tiles, block-major then slice
    static constexpr int V_STAGES = (D <= 32) ? 3 : 2;  // V tiles per slice
    static constexpr int V_CHUNKS = TILE / 16 / 32;     // 16 B chunks per lane in a V tile
    // chunks per lane the slice's helper converts (warp 3 converts the rest)
    static constexpr int V_HELPER_CHUNKS = (D == 64) ? V_CHUNKS / 2 : 0;
    static constexpr int AUG_ROW = 32;                // mask columns: 16 bf16 per row
    static constexpr int AUG_TILE = kBM * AUG_ROW;
    static constexpr int M_STAGES = 2;                // mask-column tiles per slice
    static constexpr int BIAS_BYTES = kBM * kBN * 2;  // two 128x64 boxes, 128 B swizzle
    static constexpr int B_RING = (D <= 32) ? 3 : 2;           // bias tiles in flight
    static constexpr int B_STAGES = HAS_PAIR ? B_RING : 0;      // allocated
    // shared-memory map (offsets from a 1024-aligned base; every tile 1024-aligned)
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_QAUG = OFF_Q + 2 * TILE;
    static constexpr int OFF_K = OFF_QAUG + AUG_TILE;
    static constexpr int OFF_V = OFF_K + K_STAGES * TILE;         // [2 slices][V_STAGES]
    static constexpr int OFF_ONES = OFF_V + 2 * V_STAGES * TILE;  // constant ones tile (D <= 32)
    static constexpr int OFF_KAUG = OFF_ONES + (SUM_MMA ? TILE : 0);  // [2 slices][M_STAGES]
    static constexpr int OFF_BIAS = OFF_KAUG + 2 * M_STAGES * AUG_TILE;
    static constexpr int OFF_MC = OFF_BIAS + B_STAGES * BIAS_BYTES;  // [2][M_STAGES] f32 rebase c
    static constexpr int OFF_BAR = OFF_MC + 64;
    // barrier indices
    static constexpr int BAR_Q = 0;
    static constexpr int BAR_KF = 1;                        // K tile landed
    static constexpr int BAR_KE = BAR_KF + K_STAGES;        // K tile consumed
    static constexpr int BAR_VF = BAR_KE + K_STAGES;        // [2][V_STAGES] V tile landed (bf16)
    static constexpr int BAR_VE = BAR_VF + 2 * V_STAGES;    // [2][V_STAGES] V tile consumed
    static constexpr int BAR_VC = BAR_VE + 2 * V_STAGES;    // [2][V_STAGES] V tile converted to fp16
    static constexpr int BAR_BF = BAR_VC + 2 * V_STAGES;    // [3] bias tile landed
    static constexpr int BAR_BE = BAR_BF + 3;               // [3] bias tile consumed
    static constexpr int BAR_MF = BAR_BE + 3;               // [2][M_STAGES] mask columns written
    static constexpr int BAR_ME = BAR_MF + 2 * M_STAGES;    // [2][M_STAGES] used by MMA and softmax
    static constexpr int BAR_SF = BAR_ME + 2 * M_STAGES;    // [2] S of slice w ready
    static constexpr int BAR_SE = BAR_SF + 2;               // [2] slice w has read S
    static constexpr int BAR_PF = BAR_SE + 2;               // [2] P of slice w written
    static constexpr int BAR_PE = BAR_PF + 2;               // [2] P.V of slice w done
    static constexpr int BAR_DRAIN = BAR_PE + 2;            // [2] a helper's MMAs, on abort
    static constexpr int NUM_BARS = BAR_DRAIN + 2;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;  // tmem slot, abort flag
    static constexpr int USED = OFF_MISC + 16;
    // Request at least 116 KB so that two CTAs never share an SM: each CTA
    // allocates all 512 tensor-memory columns.
    static constexpr int SMEM_BYTES = (USED + 1024 > 116 * 1024) ? USED + 1024 : 116 * 1024;
    static_assert(USED + 1024 <= 227 * 1024, "shared memory");
    // tensor-memory columns
    static constexpr uint32_t TM_S0 = 0;    // + 128 * w
    static constexpr uint32_t TM_P0 = 256;  // + 64 * w
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
    const bool aug = p.aug != 0;

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
        for (int s = 0; s < 2 * C::V_STAGES; ++s) {
            ptx::mbar_init(bar(C::BAR_VF + s), 1);
            ptx::mbar_init(bar(C::BAR_VE + s), 1);
            ptx::mbar_init(bar(C::BAR_VC + s), C::V_HELPER_CHUNKS > 0 ? 2 : 1);  // warp 3 (+ helper)
        }
        for (int s = 0; s < 3; ++s) {
            ptx::mbar_init(bar(C::BAR_BF + s), 1);
            ptx::mbar_init(bar(C::BAR_BE + s), 4 * n_valid);
        }
        for (int s = 0; s < 2 * C::M_STAGES; ++s) {
            ptx::mbar_init(bar(C::BAR_MF + s), 1);
            ptx::mbar_init(bar(C::BAR_ME + s), 1 + 4);  // the MMA's commit + 4 softmax warps
        }
        for (int w = 0; w < 2; ++w) {
            ptx::mbar_init(bar(C::BAR_SF + w), 1);
            ptx::mbar_init(bar(C::BAR_SE + w), 4);
            ptx::mbar_init(bar(C::BAR_PF + w), 4);
            ptx::mbar_init(bar(C::BAR_PE + w), 1);
        }
        ptx::mbar_init(bar(C::BAR_DRAIN + 0), 1);
        ptx::mbar_init(bar(C::BAR_DRAIN + 1), 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
        // Thread 0 is also the producer: Q and the first key block's K and bias
        // tiles go out now, before the CTA-wide setup below (their shared-memory
        // regions are not touched by it), so that their latency overlaps it.
        ptx::prefetch_tmap(&tm_q);
        ptx::prefetch_tmap(&tm_k);
        if (HAS_PAIR) ptx::prefetch_tmap(&tm_pair);
        const int bn0 = b * p.N + n0;
        ptx::mbar_arrive_expect_tx(bar(C::BAR_Q), uint32_t(n_valid * C::TILE));
        for (int w = 0; w < n_valid; ++w)
            ptx::tma_load_4d(sb + C::OFF_Q + w * C::TILE, &tm_q, bar(C::BAR_Q), 0, h, q0, bn0 + w);
        for (int w = 0; w < n_valid; ++w) {  // K stages 0 and 1 are free
            ptx::mbar_arrive_expect_tx(bar(C::BAR_KF + w), C::TILE);
            ptx::tma_load_4d(sb + C::OFF_K + w * C::TILE, &tm_k, bar(C::BAR_KF + w), 0, h, 0, bn0 + w);
        }
        if (HAS_PAIR) {  // bias stage 0 is free
            ptx::mbar_arrive_expect_tx(bar(C::BAR_BF), C::BIAS_BYTES);
            ptx::tma_load_3d(sb + C::OFF_BIAS, &tm_pair, bar(C::BAR_BF), 0, q0, bh);
            ptx::tma_load_3d(sb + C::OFF_BIAS + C::BIAS_BYTES / 2, &tm_pair, bar(C::BAR_BF), 64, q0, bh);
        }
    }
    if (warp == 1) {
        // Constant tiles.  The ones tile (D <= 32), the N-continuation of every
        // V tile in the P.V MMA: column 0 = 1.0 (fp16), rest 0.  The A tile of
        // the mask step: columns 0-2 = 1.0 (bf16), rest 0.  The mask-column B
        // tiles start zeroed; only columns 0-2 are rewritten.
        if (C::SUM_MMA)
            for (int c = lane; c < C::TILE / 16; c += 32)
                ptx::st_shared_v4(sb + C::OFF_ONES + uint32_t(c) * 16u, make_uint4(0u, 0u, 0u, 0u));
        for (int c = lane; c < (C::AUG_TILE * (1 + 2 * C::M_STAGES)) / 16; c += 32) {
            const uint32_t addr = (c < C::AUG_TILE / 16) ? sb + C::OFF_QAUG + uint32_t(c) * 16u
                                                         : sb + C::OFF_KAUG + uint32_t(c - C::AUG_TILE / 16) * 16u;
            ptx::st_shared_v4(addr, make_uint4(0u, 0u, 0u, 0u));
        }
        __syncwarp();
        if (C::SUM_MMA)
            for (int r = lane; r < kBM; r += 32)
                asm volatile("st.shared.u16 [%0], %1;" ::"r"(sb + C::OFF_ONES + swz_chunk<C::ROW>(r, 0)),
                             "h"(uint16_t(0x3C00)) : "memory");
        for (int r = lane; r < kBM; r += 32)
            ptx::st_shared_v2(sb + C::OFF_QAUG + swz_chunk<C::AUG_ROW>(r, 0), 0x3F803F80u, 0x00003F80u);
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
    if (warp < kFirstSoftmaxWarp) ptx::setmaxnreg_dec<kHelperRegs>();
    else ptx::setmaxnreg_inc<kSoftmaxRegs>();

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const int bn0 = b * p.N + n0;
            // Q, K(block 0) and bias(block 0) went out with the barrier setup.
            int k_issued = n_valid, b_issued = HAS_PAIR ? 1 : 0;
            bool ok = true;
            for (int j = 1; j < nkb && ok; ++j) {
                for (int w = 0; w < n_valid && ok; ++w) {
                    const int s = k_issued % C::K_STAGES;
                    const uint32_t ph = (k_issued / C::K_STAGES) & 1;
                    if (!wait_bounded(bar(C::BAR_KE + s), ph ^ 1, abort_flag)) { ok = false; break; }
                    ptx::mbar_arrive_expect_tx(bar(C::BAR_KF + s), C::TILE);
                    ptx::tma_load_4d(sb + C::OFF_K + s * C::TILE, &tm_k, bar(C::BAR_KF + s), 0, h, j * kBN, bn0 + w);
                    ++k_issued;
                }
                if (HAS_PAIR && ok) {
                    const int s = b_issued % C::B_RING;
                    const uint32_t ph = (b_issued / C::B_RING) & 1;
                    if (!wait_bounded(bar(C::BAR_BE + s), ph ^ 1, abort_flag)) { ok = false; break; }
                    const uint32_t dst = sb + C::OFF_BIAS + s * C::BIAS_BYTES;
                    ptx::mbar_arrive_expect_tx(bar(C::BAR_BF + s), C::BIAS_BYTES);
                    ptx::tma_load_3d(dst, &tm_pair, bar(C::BAR_BF + s), j * kBN, q0, bh);
                    ptx::tma_load_3d(dst + C::BIAS_BYTES / 2, &tm_pair, bar(C::BAR_BF + s), j * kBN + 64, q0, bh);
                    ++b_issued;
                }
            }
            if (!ok) {
                // Let every copy this thread started land before the CTA exits.
                wait_bounded(bar(C::BAR_Q), 0, nullptr);
                for (int i = (k_issued > C::K_STAGES ? k_issued - C::K_STAGES : 0); i < k_issued; ++i)
                    wait_bounded(bar(C::BAR_KF + i % C::K_STAGES), (i / C::K_STAGES) & 1, nullptr);
                for (int i = (b_issued > C::B_RING ? b_issued - C::B_RING : 0); i < b_issued; ++i)
                    wait_bounded(bar(C::BAR_BF + i % C::B_RING), (i / C::B_RING) & 1, nullptr);
            }
        }
        __syncwarp();
    } else if (warp < kFirstSoftmaxWarp) {
        // Both roles of the helper warpgroup sit under the same condition as its
        // setmaxnreg above; as separate branches of this if-chain the code
        // generator no longer held them to the smaller register budget and
        // spilled.
        if (warp == 3) {
            // ---------------------------------- V to fp16, both slices
            // Block by block, slice 0 then slice 1.  A V tile is reloaded only
            // after its P.V, which waits for this warp's conversion, so this
            // warp is never a whole ring behind the barrier phases it waits on.
            bool ok = true;
            for (int j = 0; j < nkb && ok; ++j) {
                for (int w = 0; w < n_valid && ok; ++w) {
                    const int vs = w * C::V_STAGES + j % C::V_STAGES;
                    ok = wait_warp(bar(C::BAR_VF + vs), (j / C::V_STAGES) & 1, abort_flag);
                    if (!ok) break;
                    convert_v_chunks<C::V_HELPER_CHUNKS, C::V_CHUNKS - C::V_HELPER_CHUNKS>(
                        sb + C::OFF_V + uint32_t(vs * C::TILE), lane);
                    if (lane == 0) ptx::mbar_arrive(bar(C::BAR_VC + vs));
                }
            }
        } else {
            // -------------------------------- helper of slice w: V, mask, MMAs
            // Per block j this warp issues Q K^T(j) once the softmax has pulled
            // S(j-1) into registers, writes the mask columns of block j+1, loads
            // V, and issues P.V(j-1) once warp 3 has converted V(j-1) and the
            // softmax has written P(j-1): a fixed order that follows the softmax,
            // each step a blocking wait on one barrier (no polling).  Lane 0
            // issues the MMAs.
            const int w = warp - 1;
            if (w < n_valid) {
                const uint16_t* mrow = p.mask != nullptr ? p.mask + (size_t(b) * p.N + n0 + w) * size_t(p.S) : nullptr;
                float c_run = -INFINITY;
                bool ok = true;
                // mask values of a block, fetched one block before they are needed:
                // lane l handles keys l, l+32, l+64, l+96
                uint32_t raw[4] = {0u, 0u, 0u, 0u};
                auto fetch = [&](int j) {
    #pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int key = j * kBN + lane + 32 * k;
                        raw[k] = (mrow != nullptr && key < p.S) ? uint32_t(mrow[key]) : 0u;
                    }
                };
                auto write_mask = [&](int j) -> bool {
                    float v[4];
                    float bmax = -INFINITY;
    #pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int key = j * kBN + lane + 32 * k;
                        v[k] = key < p.S ? __uint_as_float(raw[k] << 16) : -INFINITY;
                        bmax = fmaxf(bmax, v[k]);
                    }
    #pragma unroll
                    for (int o = 16; o > 0; o >>= 1) bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, o));
                    c_run = fmaxf(c_run, bmax);
                    const float csub = (c_run == -INFINITY) ? 0.f : c_run;  // all -inf so far: keep -inf logits
                    const int stage = j % C::M_STAGES;
                    const int ms = w * C::M_STAGES + stage;
                    if (!wait_warp(bar(C::BAR_ME + ms), ((j / C::M_STAGES) & 1) ^ 1, abort_flag)) return false;
                    const uint32_t tile = sb + C::OFF_KAUG + uint32_t(ms * C::AUG_TILE);
    #pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int key = lane + 32 * k;
                        // (mask - c) * sqrt(D) as hi + mid + lo, three bf16 that sum to the fp32 value
                        // A key whose mask lies more than kMaskFloor below c weighs exactly
                        // zero (e^-16384 underflows fp32 and fp64 alike): it enters as -inf, so
                        // that no logit near -1e9 ever meets a running maximum near -1e9.
                        const float x = (v[k] - csub < -kMaskFloor) ? -INFINITY : (v[k] - csub) * p.sqrt_d;
                        const uint32_t hi = ptx::f32_to_bf16_bits(x);
                        uint32_t mid = 0, lo = 0;
                        if (fabsf(x) < INFINITY) {
                            const float r1 = x - __uint_as_float(hi << 16);
                            mid = ptx::f32_to_bf16_bits(r1);
                            lo = ptx::f32_to_bf16_bits(r1 - __uint_as_float(mid << 16));
                        }
                        ptx::st_shared_v2(tile + swz_chunk<C::AUG_ROW>(key, 0), hi | (mid << 16), lo);
                    }
                    if (lane == 0) mc_s[ms] = csub;
                    ptx::fence_proxy_async_smem();  // generic-proxy writes -> tensor-core reads
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(bar(C::BAR_MF + ms));
                    return true;
                };
                // This warp loads the slice's V tiles itself (lane 0), V_STAGES ahead,
                // so that V never waits behind K or the bias in another thread's queue.
                const int bn = b * p.N + n0 + w;
                int v_issued = 0;
                auto load_v = [&](int j) -> bool {
                    const int vs = w * C::V_STAGES + j % C::V_STAGES;
                    // the tile's previous block (j - V_STAGES) must be consumed by its P.V
                    if (!wait_warp(bar(C::BAR_VE + vs), ((j / C::V_STAGES) & 1) ^ 1, abort_flag)) return false;
                    if (lane == 0) {
                        ptx::mbar_arrive_expect_tx(bar(C::BAR_VF + vs), C::TILE);
                        ptx::tma_load_4d(sb + C::OFF_V + vs * C::TILE, &tm_v, bar(C::BAR_VF + vs), 0, h, j * kBN, bn);
                    }
                    v_issued = j + 1;
                    return true;
                };
                // D = 64: the first half of V tile j to fp16 (warp 3 converts the rest)
                auto convert_v = [&](int j) -> bool {
                    if (C::V_HELPER_CHUNKS == 0) return true;
                    const int vs = w * C::V_STAGES + j % C::V_STAGES;
                    if (!wait_warp(bar(C::BAR_VF + vs), (j / C::V_STAGES) & 1, abort_flag)) return false;
                    convert_v_chunks<0, C::V_HELPER_CHUNKS>(sb + C::OFF_V + uint32_t(vs * C::TILE), lane);
                    if (lane == 0) ptx::mbar_arrive(bar(C::BAR_VC + vs));
                    return true;
                };
                const uint32_t d_s = tmem + C::TM_S0 + 128u * w;
                const uint32_t d_o = tmem + C::TM_O0 + uint32_t(C::OW) * w;
                const uint32_t a_p = tmem + C::TM_P0 + 64u * w;
                const uint64_t a_q = desc_k_major<C::ROW>(sb + C::OFF_Q + w * C::TILE);
                bool issued_any = false;
                auto issue_qk = [&](int j) -> bool {
                    const int ki = j * n_valid + w;  // the producer's K tile order
                    const int ks = ki % C::K_STAGES;
                    if (!wait_warp(bar(C::BAR_KF + ks), (ki / C::K_STAGES) & 1, abort_flag)) return false;
                    if (lane == 0) {
                        ptx::tc_fence_after();
                        const uint64_t bd = desc_k_major<C::ROW>(sb + C::OFF_K + ks * C::TILE);
    #pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk)  // 16 bf16 = 32 B per K step
                            ptx::mma_ss(d_s, a_q + uint64_t(2 * kk), bd + uint64_t(2 * kk), C::IDESC_QK, kk > 0 ? 1u : 0u);
                        if (aug) {
                            const int ms = w * C::M_STAGES + j % C::M_STAGES;
                            ptx::mma_ss(d_s, desc_k_major<C::AUG_ROW>(sb + C::OFF_QAUG),
                                        desc_k_major<C::AUG_ROW>(sb + C::OFF_KAUG + ms * C::AUG_TILE), C::IDESC_QK, 1u);
                            ptx::mma_commit(bar(C::BAR_ME + ms));
                        }
                        ptx::mma_commit(bar(C::BAR_KE + ks));
                        ptx::mma_commit(bar(C::BAR_SF + w));
                    }
                    issued_any = true;
                    __syncwarp();
                    return true;
                };
                auto issue_pv = [&](int j) -> bool {
                    // P(j) written by the four softmax warps; V(j) converted by warp 3 (and this warp)
                    const int vs = w * C::V_STAGES + j % C::V_STAGES;
                    if (!wait_warp(bar(C::BAR_VC + vs), (j / C::V_STAGES) & 1, abort_flag)) return false;
                    if (!wait_warp(bar(C::BAR_PF + w), j & 1, abort_flag)) return false;
                    if (lane == 0) {
                        ptx::tc_fence_after();
                        const uint32_t v_off = uint32_t(C::OFF_V + vs * C::TILE);
                        // the ones tile continues V along N (D <= 32); unused for D = 64
                        const uint64_t bd =
                            desc_mn_major<C::ROW>(sb + v_off, C::SUM_MMA ? uint32_t(C::OFF_ONES) - v_off : uint32_t(C::TILE));
    #pragma unroll
                        for (int kk = 0; kk < kBN / 16; ++kk)  // 16 keys per K step = 16 rows of V
                            ptx::mma_ts(d_o, a_p + 8u * kk, bd + uint64_t((16 * C::ROW * kk) >> 4), C::IDESC_PV,
                                        (j > 0 || kk > 0) ? 1u : 0u);
                        ptx::mma_commit(bar(C::BAR_VE + vs));
                        ptx::mma_commit(bar(C::BAR_PE + w));
                    }
                    __syncwarp();
                    return true;
                };
                if (lane == 0) ptx::prefetch_tmap(&tm_v);
                // V(0) and V(1) go out first; later V(j+1) is loaded in iteration j,
                // into the tile that P.V(j+1-V_STAGES) has released.
                for (int j = 0; j < 2 && j < nkb && ok; ++j) ok = load_v(j);
                if (aug && ok) {
                    fetch(0);
                    for (int j = 0; j < C::M_STAGES && j < nkb && ok; ++j) {
                        ok = write_mask(j);
                        fetch(j + 1);
                    }
                }
                ok = ok && wait_warp(bar(C::BAR_Q), 0, abort_flag);
                ok = ok && issue_qk(0);
                ok = ok && convert_v(0);
                for (int j = 1; j <= nkb && ok; ++j) {
                    if (j < nkb) {
                        // S(j-1) is in the softmax's registers: Q K^T(j) may overwrite it
                        ok = wait_warp(bar(C::BAR_SE + w), (j - 1) & 1, abort_flag) && issue_qk(j);
                        if (ok && aug && j + 1 < nkb) {
                            ok = write_mask(j + 1);
                            fetch(j + 2);
                        }
                        if (ok && C::V_STAGES >= 3 && j + 1 < nkb) ok = load_v(j + 1);
                        ok = ok && convert_v(j);
                    }
                    ok = ok && issue_pv(j - 1);
                    if (ok && C::V_STAGES < 3 && j + 1 < nkb) ok = load_v(j + 1);
                }
                if (!ok && lane == 0) {
                    // Wait for every MMA and V copy this warp started before the CTA
                    // frees tensor memory and exits.
                    if (issued_any) {
                        ptx::mma_commit(bar(C::BAR_DRAIN + w));
                        wait_bounded(bar(C::BAR_DRAIN + w), 0, nullptr);
                    }
                    for (int i = (v_issued > C::V_STAGES ? v_issued - C::V_STAGES : 0); i < v_issued; ++i)
                        wait_bounded(bar(C::BAR_VF + w * C::V_STAGES + i % C::V_STAGES), (i / C::V_STAGES) & 1, nullptr);
                }
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax
        const int w = (warp - kFirstSoftmaxWarp) >> 2;  // slice (n0 + w)
        const int quarter = warp & 3;                   // TMEM lanes 32*quarter .. +31
        const int r = quarter * 32 + lane;              // query row in the tile == TMEM lane
        if (w < n_valid) {
            const uint32_t lane_base = uint32_t(quarter * 32) << 16;
            const uint32_t tS = tmem + lane_base + C::TM_S0 + 128u * w;
            const uint32_t tP = tmem + lane_base + C::TM_P0 + 64u * w;
            const uint32_t tO = tmem + lane_base + C::TM_O0 + uint32_t(C::OW) * w;
            const float2 sqd2 = make_float2(p.sqrt_d, p.sqrt_d);
            const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
            float m_used = -INFINITY;
            float c_cur = 0.f;  // mask rebase the current m_used and P are relative to
            float l = 0.f;      // row sum when the tensor core does not keep it
            bool ok = true;
            // Bias of chunk c (keys 8c .. 8c+7) of this row, as the fp32 pair
            // bias * sqrt(D) for keys (8c + 2e, 8c + 2e + 1): the tile is two
            // 128 x 64 boxes with the 128 B swizzle, so chunk (c % 8) of row r
            // in box c / 8 sits at chunk (c % 8) ^ (r % 8) of the row.
            auto bias_row = [&](int bstage) -> uint32_t {
                return (sb + C::OFF_BIAS + uint32_t(bstage * C::BIAS_BYTES) + uint32_t(r * 128)) |
                       uint32_t((r & 7) << 4);
            };
            auto bias_chunk = [&](uint32_t brow, int c) -> uint4 {
                return ptx::ld_shared_v4((brow ^ uint32_t((c & 7) << 4)) + uint32_t((c >> 3) * (C::BIAS_BYTES / 2)));
            };
            // t = S + bias * sqrt(D) for keys k, k + 1 (in place in s), and the running maxima
            auto add_bias = [&](uint32_t* s, int k, uint32_t word, float& rmax) {
                const float2 t = __ffma2_rn(make_float2(ptx::bf16lo_to_f32(word), ptx::bf16hi_to_f32(word)), sqd2,
                                            make_float2(__uint_as_float(s[k]), __uint_as_float(s[k + 1])));
                s[k] = __float_as_uint(t.x);
                s[k + 1] = __float_as_uint(t.y);
                rmax = max3f(rmax, t.x, t.y);
            };
            // p = 2^(t * log2(e) / sqrt(D) - m) for keys k, k + 1, packed as fp16
            auto exp_pair = [&](const uint32_t* s, int k, float2 nm2, float2& acc) -> uint32_t {
                const float2 x = __ffma2_rn(make_float2(__uint_as_float(s[k]), __uint_as_float(s[k + 1])), sc2, nm2);
                const float p0 = ptx::ex2_approx(x.x);
                const float p1 = ptx::ex2_approx(x.y);
                if (!C::SUM_MMA) acc = __fadd2_rn(acc, make_float2(p0, p1));
                return ptx::pack_f16x2(p0, p1);  // P column k/2 holds keys k (low) and k+1
            };
            auto rescale_o = [&](float alpha) {
#pragma unroll
                for (int dc = 0; dc < C::OW; dc += 16) {
                    uint32_t o[16];
                    ptx::tmem_ld_x16(tO + dc, o);
                    ptx::tmem_ld_wait_x16(o);
#pragma unroll
                    for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                    ptx::tmem_st_x16(tO + dc, o);
                }
            };
            uint32_t s[128];  // s[i] = S[r][i] of the current block
            // S(j) is loaded while the block's other inputs are waited for; from
            // the second block on it was requested at the end of the previous one.
            auto load_s = [&](int j) -> bool {
                if (!wait_warp(bar(C::BAR_SF + w), j & 1, abort_flag)) return false;
                ptx::tc_fence_after();
                ptx::tmem_ld_x32(tS + 0, s);
                ptx::tmem_ld_x32(tS + 32, s + 32);
                ptx::tmem_ld_x32(tS + 64, s + 64);
                ptx::tmem_ld_x32(tS + 96, s + 96);
                return true;
            };
            for (int j = 0; j < nkb && ok; ++j) {
                ok = load_s(j);
                if (!ok) break;
                float cs = c_cur;
                if (aug) {
                    const int ms = w * C::M_STAGES + j % C::M_STAGES;
                    ok = wait_warp(bar(C::BAR_MF + ms), (j / C::M_STAGES) & 1, abort_flag);
                    if (!ok) break;
                    cs = mc_s[ms];
                    ptx::mbar_arrive_elect(bar(C::BAR_ME + ms));
                }
                const int bstage = j % C::B_RING;
                uint32_t brow = 0;
                if (HAS_PAIR) {
                    ok = wait_warp(bar(C::BAR_BF + bstage), (j / C::B_RING) & 1, abort_flag);
                    if (!ok) break;
                    brow = bias_row(bstage);
                }
                ptx::tmem_ld_wait_x32(s);
                ptx::reg_fence_x32(s + 32);
                ptx::reg_fence_x32(s + 64);
                ptx::reg_fence_x32(s + 96);
                ptx::tc_fence_before();
                ptx::mbar_arrive_elect(bar(C::BAR_SE + w));
                if (cs != c_cur) {
                    // the mask rebase grew: earlier logits are relative to a smaller c
                    m_used -= (cs - c_cur) * kLog2e;
                    c_cur = cs;
                }
                // P.V of block j - 1 must be done before P is overwritten and O rescaled
                auto wait_pv = [&]() -> bool {
                    if (j == 0) return true;
                    if (!wait_warp(bar(C::BAR_PE + w), (j - 1) & 1, abort_flag)) return false;
                    ptx::tc_fence_after();
                    return true;
                };
                float2 acc = make_float2(0.f, 0.f);
                float alpha = 1.f;
                float rmax0 = -INFINITY, rmax1 = -INFINITY;
                if (__any_sync(0xffffffffu, m_used == -INFINITY)) {
                    // No running maximum yet (first block, or every key so far -inf):
                    // pass 1 finds the block maximum, pass 2 exponentiates.
                    if (HAS_PAIR) {
#pragma unroll
                        for (int c = 0; c < 16; ++c) {
                            const uint4 pw = bias_chunk(brow, c);
                            add_bias(s, 8 * c + 0, pw.x, rmax0);
                            add_bias(s, 8 * c + 2, pw.y, rmax1);
                            add_bias(s, 8 * c + 4, pw.z, rmax0);
                            add_bias(s, 8 * c + 6, pw.w, rmax1);
                        }
                        ptx::mbar_arrive_elect(bar(C::BAR_BE + bstage));
                    } else {
#pragma unroll
                        for (int k = 0; k < 128; k += 4) {
                            rmax0 = max3f(rmax0, __uint_as_float(s[k]), __uint_as_float(s[k + 1]));
                            rmax1 = max3f(rmax1, __uint_as_float(s[k + 2]), __uint_as_float(s[k + 3]));
                        }
                    }
                    const float m_new = fmaxf(m_used, fmaxf(rmax0, rmax1) * p.scale_log2);
                    if (m_new > m_used) {
                        alpha = ptx::ex2_approx(m_used - m_new);  // 0 while m_used is -inf
                        m_used = m_new;
                    }
                    const float m_safe = (m_used == -INFINITY) ? 0.f : m_used;
                    const float2 nm2 = make_float2(-m_safe, -m_safe);
                    ok = wait_pv();
                    if (!ok) break;
                    if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) rescale_o(alpha);
#pragma unroll
                    for (int c = 0; c < 8; ++c) {  // 16 keys -> 8 P columns per store
                        uint32_t pk[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) pk[e] = exp_pair(s, 16 * c + 2 * e, nm2, acc);
                        ptx::tmem_st_x8(tP + 8u * c, pk);
                    }
                } else {
                    // One pass against the running maximum m: t, its maximum and
                    // p = 2^(t - m) together, so the exp unit is busy from the
                    // start of the block.  p <= 2^12 unless the block raises the
                    // maximum by more than 12; then P is recomputed below.
                    const float2 nm2 = make_float2(-m_used, -m_used);
                    // The first kHeldChunks chunks of P stay in registers, so that the
                    // wait for P.V(j-1) (which still reads the P buffer) comes a few
                    // chunks into the pass, when that P.V has usually finished.
                    constexpr int kHeldChunks = 3;
                    uint32_t held[kHeldChunks][8];
#pragma unroll
                    for (int c = 0; c < 8; ++c) {  // 16 keys -> 8 P columns per store
                        uint32_t pk_own[8];
                        uint32_t* pk = c < kHeldChunks ? held[c < kHeldChunks ? c : 0] : pk_own;
#pragma unroll
                        for (int q = 0; q < 2; ++q) {
                            const int k = 16 * c + 8 * q;
                            if (HAS_PAIR) {
                                const uint4 pw = bias_chunk(brow, 2 * c + q);
                                add_bias(s, k + 0, pw.x, rmax0);
                                add_bias(s, k + 2, pw.y, rmax1);
                                add_bias(s, k + 4, pw.z, rmax0);
                                add_bias(s, k + 6, pw.w, rmax1);
                            } else {
                                rmax0 = max3f(rmax0, __uint_as_float(s[k]), __uint_as_float(s[k + 1]));
                                rmax1 = max3f(rmax1, __uint_as_float(s[k + 2]), __uint_as_float(s[k + 3]));
                                rmax0 = max3f(rmax0, __uint_as_float(s[k + 4]), __uint_as_float(s[k + 5]));
                                rmax1 = max3f(rmax1, __uint_as_float(s[k + 6]), __uint_as_float(s[k + 7]));
                            }
#pragma unroll
                            for (int e = 0; e < 4; ++e) pk[4 * q + e] = exp_pair(s, k + 2 * e, nm2, acc);
                        }
                        if (c < kHeldChunks) continue;  // computed straight into held[c]
                        if (c == kHeldChunks) {
                            ok = wait_pv();
                            if (!ok) break;
#pragma unroll
                            for (int h2 = 0; h2 < kHeldChunks; ++h2) ptx::tmem_st_x8(tP + 8u * h2, held[h2]);
                        }
                        ptx::tmem_st_x8(tP + 8u * c, pk);
                    }
                    if (!ok) break;
                    if (HAS_PAIR) ptx::mbar_arrive_elect(bar(C::BAR_BE + bstage));
                    const float m_blk = fmaxf(rmax0, rmax1) * p.scale_log2;
                    const bool raise = m_blk > m_used + kRescaleThreshold;
                    if (__any_sync(0xffffffffu, raise)) {
                        // Rare: P overflows the fp16 headroom.  Move m to the block
                        // maximum, rescale O, recompute P from t (still in s).
                        if (raise) {
                            alpha = ptx::ex2_approx(m_used - m_blk);
                            m_used = m_blk;
                        }
                        const float2 nm2b = make_float2(-m_used, -m_used);
                        ptx::tmem_st_wait();
                        rescale_o(alpha);
                        acc = make_float2(0.f, 0.f);
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            uint32_t pk[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e) pk[e] = exp_pair(s, 16 * c + 2 * e, nm2b, acc);
                            ptx::tmem_st_x8(tP + 8u * c, pk);
                        }
                    }
                }
                if (!C::SUM_MMA) l = l * alpha + (acc.x + acc.y);
                ptx::tmem_st_wait();
                ptx::tc_fence_before();
                ptx::mbar_arrive_elect(bar(C::BAR_PF + w));
            }
            // ---------------------------------------------------------- epilogue
            if (ok) ok = wait_warp(bar(C::BAR_PE + w), (nkb - 1) & 1, abort_flag);
            if (ok) {
                ptx::tc_fence_after();
                const int n = n0 + w;
                const int row = q0 + r;
                uint32_t o[C::OW];  // 32, 48 or 64 columns
                ptx::tmem_ld_x32(tO, o);
                if constexpr (C::OW == 48) ptx::tmem_ld_x16(tO + 32, o + 32);
                if constexpr (C::OW == 64) ptx::tmem_ld_x32(tO + 32, o + 32);
                ptx::tmem_ld_wait_x32(o);
                if constexpr (C::OW == 48) {
                    ptx::reg_fence_x8(o + 32);
                    ptx::reg_fence_x8(o + 40);
                }
                if constexpr (C::OW == 64) ptx::reg_fence_x32(o + 32);
                if (C::SUM_MMA) l = __uint_as_float(o[D]);  // column D holds the row sum
                const float inv_l = l > 0.f ? 1.f / l : 0.f;
                bool finite = (l < INFINITY);  // an fp16 overflow of V shows up here or in O
                if (row < p.S) {
                    uint16_t* orow =
                        p.out + ((size_t(b) * p.N + n) * size_t(p.S) + size_t(row)) * size_t(p.H) * D + size_t(h) * D;
#pragma unroll
                    for (int k = 0; k < D; k += 8) {
                        float f[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            f[e] = __uint_as_float(o[k + e]) * inv_l;
                            finite = finite && fabsf(f[e]) < INFINITY;
                        }
                        uint4 v;
                        v.x = ptx::pack_bf16x2(f[0], f[1]);
                        v.y = ptx::pack_bf16x2(f[2], f[3]);
                        v.z = ptx::pack_bf16x2(f[4], f[5]);
                        v.w = ptx::pack_bf16x2(f[6], f[7]);
                        *reinterpret_cast<uint4*>(orow + k) = v;
                    }
                    if (!finite) record_status(EVO_ERR_RANGE);
                    const float lse = l > 0.f ? (m_used + ptx::lg2_approx(l)) * kLn2 + c_cur : -INFINITY;
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
