// bf16 biased-attention forward on sm_100a for head dims 16 and 32: three n
// slices per tile, persistent CTAs, P written over the scores it came from.
//
// What it computes is the forward pass of the DeepSpeed DS4Sci_EvoformerAttention
// guide (hmyw.cn): section 4's softmax(Q K^T * scale + biases) V with section
// 5.2's bias shapes and section 5.4's log-sum-exp.  The design is Blackwell's:
//
//  * A tile is one (b, h, 128-query block) and THREE n slices, n0 .. n0+2.  The
//    pair bias [B,1,H,S,S] does not depend on n, so the three slices read one
//    128x128 bias tile from shared memory (one L2->SM transfer feeds three
//    softmax warpgroups).  Tiles are numbered query block fastest, then head,
//    then n triple, then batch; a grid of one CTA per SM walks them with a
//    stride of the grid size, so the tiles that share one (n, h) K/V slice run
//    at the same time and hit L2.
//  * Warp roles (512 threads): warp 0 loads the shared bias tiles and writes
//    the mask columns of every slice; warp 1 + w drives slice w: its Q, K and
//    V loads, the conversion of its V tiles to fp16 and its tcgen05 MMAs,
//    issued by one elected lane of the converged warp (a tensor-core
//    instruction keeps its issuing warp busy for about a hundred cycles, so
//    each slice has its own issuer); warps 4-7, 8-11 and 12-15 are the
//    softmax warpgroups of slices 0, 1, 2 (warp w reads tensor-memory lanes
//    32 (w % 4) ..).  A softmax thread owns one query row.
//  * Tensor memory (512 columns): per slice a 128-column score buffer S and
//    a D-column O accumulator.  The softmax writes P (fp16) over the first 64
//    columns of S, 16 keys' worth at a time, each over scores it has already
//    read.  The MMA warp issues P.V(j) and then Q K^T(j+1) of the same slice
//    into the same columns; tcgen05 MMAs of one thread run in issue order, so
//    S(j+1) lands after P(j) was read, and the commit that signals S(j+1)
//    also proves P.V(j) complete: the softmax may rescale O at any time during
//    a block and never waits for P.V.  The last block of a tile is followed at
//    once by Q K^T of the slice's first block of the next tile.  (The MMA
//    order of one slice is P.V(j), Q K^T(j+1), ...; the slices' MMAs
//    interleave on the tensor core.)
//  * The mask bias enters through the tensor core as one more K=16 step of the
//    score MMA (A: 1, 1, 1 in columns 0-2 of every query row; B: three bf16
//    numbers per key that sum exactly to the fp32 (mask - c) * sqrt(D), c the
//    running mask maximum of the slice; keys past S get -inf).
//  * Softmax in base 2, 32 keys per step: t = S + pair * sqrt(D) (packed fp32
//    FMA), p = 2^(t log2(e) / sqrt(D) - m) against the running maximum m, P
//    packed to fp16 and stored, the row sum accumulated in registers.  m only
//    moves when a step exceeds it by more than 15 (p stays <= 2^15, inside
//    fp16; the result is exact after the division by the row sum).  The step's
//    p sum tells: at most 2^15, no p of the step is above it, so the step
//    maximum is only formed when the sum is larger.  When m moves, the P
//    already stored for the block and the O accumulator are rescaled in
//    tensor memory.  The first step of a tile always sets m this way.
//  * Every wait is bounded (about two seconds); on expiry the CTA records
//    EVO_ERR_TIMEOUT, drains its own in-flight copies and MMAs, frees tensor
//    memory and exits.
#pragma once

#include <cuda.h>
#include <cstdint>

#include "common.cuh"
#include "ptx_sm100.cuh"
#include "tile_sm100.cuh"  // descriptors, swizzle helpers, V conversion

namespace evo {

struct TriParams {
    const uint16_t* mask;  // [B, N, S] bf16 bits, or nullptr
    // [B, H, S, S] bf16 bits, read by the softmax threads straight from global
    // memory, when its rows are not whole 16-byte units (S % 8 != 0) and the
    // tensor-memory accelerator cannot load them; else nullptr (the bias
    // tiles come through the TMA ring)
    const uint16_t* pair_g;
    uint16_t* out;         // [B, N, S, H, D] bf16 bits
    float* lse;            // [B, N, H, S]
    int N, S, H;
    int num_kb;            // key blocks of 128
    int num_qb;            // query blocks of 128
    int num_ng;            // n groups per batch entry, ceil(N / slices per tile)
    int num_tiles;         // B * num_ng * H * num_qb
    int aug;               // mask columns in the score MMA (a mask, or a ragged last key block)
    float scale_log2;      // log2(e) / sqrt(D)
    float sqrt_d;          // sqrt(D)
};

// The running maximum moves when a step exceeds it by more than this (log2
// units): p <= 2^15 keeps P inside fp16 (largest finite 65504).
constexpr float kTriRescaleThreshold = 15.0f;
// A step's p sum above this (2^kTriRescaleThreshold) may hold a p past the
// threshold; at or below it none does.
constexpr float kStepSumLimit = 32768.0f;

// Slices per tile: as many as tensor memory holds, each a 128-column score
// buffer plus a D-column O accumulator.
__host__ __device__ constexpr int tri_slices(int D) { return D <= 32 ? 3 : (D == 64 ? 2 : 1); }

template <int D, bool HAS_PAIR, bool F16 = false>
struct TriCfg {
    static_assert(D == 16 || D == 32 || D == 64 || D == 128, "head dim");
    static constexpr int NS = tri_slices(D);          // slices per tile
    static constexpr int THREADS = 128 * (1 + NS);    // helper warpgroup + one softmax warpgroup per slice
    // register split (setmaxnreg) where the launch leaves less than the
    // softmax needs: the helper warpgroup hands registers to the softmax
    static constexpr bool SPLIT_REGS = NS >= 2;
    static constexpr int HELPER_REGS = NS == 3 ? 72 : 136;
    static constexpr int SOFTMAX_REGS = NS == 3 ? 144 : 176;
    static_assert(!SPLIT_REGS || 128 * HELPER_REGS + NS * 128 * SOFTMAX_REGS <= THREADS * (65536 / THREADS / 8 * 8),
                  "register split");
    // a Q/K/V row is D bf16; rows wider than 128 B are split into sub-tiles of
    // 64 elements (one 128 B swizzle atom each)
    static constexpr int SUBW = D <= 64 ? D : 64;     // elements per sub-tile row
    static constexpr int NSUB = D / SUBW;             // sub-tiles per tile
    static constexpr int ROW = SUBW * 2;              // bytes per sub-tile row = swizzle span
    static constexpr int SUBTILE = kBM * ROW;
    static constexpr int TILE = NSUB * SUBTILE;       // one Q, K or V tile
    static constexpr int KPA = SUBW / 16;             // 16-element MMA K steps per swizzle atom
    // stages per slice, as many as shared memory holds
    static constexpr int Q_BUFS = D <= 32 ? 2 : 1;    // 2: this tile's Q and the next one's
    static constexpr int K_STAGES = 2;
    static constexpr int V_STAGES = D <= 32 ? 2 : 1;
    static constexpr int V_CHUNKS = TILE / 16 / 32;   // 16 B chunks per lane of a V tile
    static constexpr int AUG_ROW = 32;                // mask columns: 16 bf16 per row
    static constexpr int AUG_TILE = kBM * AUG_ROW;
    static constexpr int M_STAGES = 1;                // mask-column tiles per slice
    static constexpr int BIAS_BYTES = kBM * kBN * 2;  // two 128x64 boxes, 128 B swizzle
    static constexpr int B_STAGES = HAS_PAIR ? 2 : 0;
    static constexpr int B_RING = HAS_PAIR ? 2 : 1;   // ring arithmetic (no bias tiles without a pair bias)
    // shared-memory map (offsets from a 1024-aligned base; every tile 1024-aligned)
    static constexpr int OFF_Q = 0;                                        // [NS][Q_BUFS]
    static constexpr int OFF_QAUG = OFF_Q + NS * Q_BUFS * TILE;
    static constexpr int OFF_K = OFF_QAUG + AUG_TILE;                      // [NS][K_STAGES]
    static constexpr int OFF_V = OFF_K + NS * K_STAGES * TILE;     // [NS][V_STAGES]
    static constexpr int OFF_KAUG = OFF_V + NS * V_STAGES * TILE;  // [NS][M_STAGES]
    static constexpr int OFF_BIAS = OFF_KAUG + NS * M_STAGES * AUG_TILE;
    static constexpr int OFF_MC = OFF_BIAS + B_STAGES * BIAS_BYTES;        // [NS][M_STAGES] f32 rebase c
    static constexpr int OFF_BAR = OFF_MC + 64;
    // barrier indices (per slice w unless noted)
    static constexpr int BAR_QF = 0;                                       // [NS][Q_BUFS] Q tile landed
    static constexpr int BAR_KF = BAR_QF + NS * Q_BUFS;            // [NS][K_STAGES] K landed
    static constexpr int BAR_KE = BAR_KF + NS * K_STAGES;          // [NS][K_STAGES] Q K^T done
    static constexpr int BAR_VF = BAR_KE + NS * K_STAGES;          // [NS][V_STAGES] V landed (bf16)
    static constexpr int BAR_VE = BAR_VF + NS * V_STAGES;          // [NS][V_STAGES] P.V done
    static constexpr int BAR_BF = BAR_VE + NS * V_STAGES;          // [2] bias tile landed (shared)
    static constexpr int BAR_BE = BAR_BF + 2;                              // [2] bias tile read by 12 softmax warps
    static constexpr int BAR_MF = BAR_BE + 2;                              // [NS][M_STAGES] mask columns written
    static constexpr int BAR_ME = BAR_MF + NS * M_STAGES;          // [NS][M_STAGES] read by MMA + softmax
    static constexpr int BAR_SF = BAR_ME + NS * M_STAGES;          // [NS][2] S of keys 0-63 / 64-127 ready
    static constexpr int BAR_PF = BAR_SF + 2 * NS;                 // [NS][2] P of keys 0-63 / 64-127 written
    static constexpr int BAR_OA = BAR_PF + 2 * NS;                 // [NS] P.V of keys 0-63 done
    static constexpr int BAR_PE = BAR_OA + NS;                     // [NS] last P.V of a tile done
    static constexpr int BAR_DRAIN = BAR_PE + NS;                  // [NS] a helper's MMAs, on abort
    static constexpr int NUM_BARS = BAR_DRAIN + NS;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;    // tmem slot, abort flag
    static constexpr int USED = OFF_MISC + 16;
    // + alignment slack; at least 116 KB so that two CTAs never share an SM
    // (each allocates all 512 tensor-memory columns)
    static constexpr int SMEM_BYTES = (USED + 1024 > 116 * 1024) ? USED + 1024 : 116 * 1024;
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
    // tensor-memory columns
    static constexpr uint32_t TM_S0 = 0;    // + 128 * w: S, with P over its first 64 columns
    static constexpr uint32_t TM_O0 = 128u * NS;  // + D * w
    static constexpr uint32_t TMEM_COLS = (TM_O0 + NS * D) <= 256 ? 256u : 512u;
    static_assert(TM_O0 + NS * D <= TMEM_COLS, "tensor memory");
    // instruction descriptors, fp32 accumulate, M = 128
    // Q K^T of one half block: bf16 x bf16 (or fp16 x fp16), both K-major,
    // N = 64 keys; the mask step is always bf16 x bf16
    static constexpr uint32_t IDESC_MASK =
        (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t(kBN / 2) >> 3) << 17) | ((uint32_t(kBM) >> 4) << 24);
    static constexpr uint32_t IDESC_QK = F16 ? (IDESC_MASK & ~((1u << 7) | (1u << 10))) : IDESC_MASK;
    static constexpr uint32_t IDESC_PV =
        (1u << 4) | (0u << 7) | (0u << 10) | (1u << 16) | ((uint32_t(D) >> 3) << 17) | ((uint32_t(kBM) >> 4) << 24);
};

// Tile coordinates of a linear tile index (query block fastest).
struct TriTile {
    int qb, h, n0, b, nv;
};

__device__ __forceinline__ TriTile tri_tile(const TriParams& p, int L, int ns) {
    TriTile t;
    t.qb = L % p.num_qb;
    int rest = L / p.num_qb;
    t.h = rest % p.H;
    rest /= p.H;
    const int ng = rest % p.num_ng;
    t.b = rest / p.num_ng;
    t.n0 = ns * ng;
    t.nv = (p.N - t.n0) < ns ? (p.N - t.n0) : ns;
    return t;
}

// One 16-bit element (bf16 or fp16 bits) -> fp32, exact.
template <bool F16>
__device__ __forceinline__ float elem_to_f32(uint32_t bits) {
    if constexpr (F16) return __half2float(__ushort_as_half(uint16_t(bits)));
    else return __uint_as_float(bits << 16);
}
// A pair of 16-bit elements in one word (lower index in the low half) -> fp32 x 2.
template <bool F16>
__device__ __forceinline__ float2 pair_to_f32x2(uint32_t w) {
    if constexpr (F16) {
        const __half2 h = *reinterpret_cast<const __half2*>(&w);
        return __half22float2(h);
    } else {
        return make_float2(ptx::bf16lo_to_f32(w), ptx::bf16hi_to_f32(w));
    }
}
// t = b * q + s for the two bf16 numbers of one 32-bit word (low half first),
// packed fp32: the word's halves become the fp32 pair in place (a shift and a
// mask) and feed one packed FMA.
__device__ __forceinline__ float2 bf16x2_fma2(uint32_t w, float2 q, float2 s) {
    unsigned long long d;
    asm("{\n\t.reg .b32 lo, hi;\n\t.reg .b64 bb, ss, qq;\n\t"
        "shl.b32 lo, %1, 16;\n\tand.b32 hi, %1, 0xffff0000;\n\t"
        "mov.b64 bb, {lo, hi};\n\tmov.b64 ss, {%2, %3};\n\tmov.b64 qq, {%4, %5};\n\t"
        "fma.rn.f32x2 %0, bb, qq, ss;\n\t}"
        : "=l"(d)
        : "r"(w), "f"(s.x), "f"(s.y), "f"(q.x), "f"(q.y));
    return make_float2(__uint_as_float(uint32_t(d)), __uint_as_float(uint32_t(d >> 32)));
}
// Two fp32 -> the output type, round to nearest even; `lo` in the low half.
template <bool F16>
__device__ __forceinline__ uint32_t pack_out(float lo, float hi) {
    if constexpr (F16) return ptx::pack_f16x2(lo, hi);
    else return ptx::pack_bf16x2(lo, hi);
}

__device__ __forceinline__ void tmem_ld_x32f(uint32_t taddr, float* f) {
    ptx::tmem_ld_x32(taddr, reinterpret_cast<uint32_t*>(f));
}
__device__ __forceinline__ void tmem_wait_x32f(float* f) { ptx::tmem_ld_wait_x32(reinterpret_cast<uint32_t*>(f)); }

// F16: Q, K, V, biases and O in fp16 instead of bf16 (V then needs no
// conversion for the P.V product, which is fp16 x fp16 either way).
template <int D, bool HAS_PAIR, bool F16>
__global__ void __launch_bounds__(TriCfg<D, HAS_PAIR, F16>::THREADS, 1)
evo_fwd_tri_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_pair,
                   const TriParams p) {
    using C = TriCfg<D, HAS_PAIR, F16>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = ptx::smem_u32(smem);

    // the warp index through a shuffle from lane 0: provably warp-uniform, so
    // the tensor-memory addresses derived from it stay in uniform registers
    const int warp = __shfl_sync(0xffffffffu, int(threadIdx.x >> 5), 0);
    const int lane = threadIdx.x & 31;
    const int nkb = p.num_kb;
    const bool aug = p.aug != 0;
    const int G = gridDim.x;
    const int first_tile = blockIdx.x;

    auto bar = [&](int i) -> uint32_t { return sb + C::OFF_BAR + 8u * uint32_t(i); };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
    float* mc_s = reinterpret_cast<float*>(smem + C::OFF_MC);  // [w * M_STAGES + stage]

    if (threadIdx.x == 0) {
        for (int w = 0; w < C::NS; ++w) {
            for (int qb = 0; qb < C::Q_BUFS; ++qb) ptx::mbar_init(bar(C::BAR_QF + w * C::Q_BUFS + qb), 1);
            for (int st = 0; st < C::K_STAGES; ++st) {
                ptx::mbar_init(bar(C::BAR_KF + w * C::K_STAGES + st), 1);
                ptx::mbar_init(bar(C::BAR_KE + w * C::K_STAGES + st), 1);
            }
            for (int st = 0; st < C::V_STAGES; ++st) {
                ptx::mbar_init(bar(C::BAR_VF + w * C::V_STAGES + st), 1);
                ptx::mbar_init(bar(C::BAR_VE + w * C::V_STAGES + st), 1);
            }
            for (int st = 0; st < C::M_STAGES; ++st) {
                ptx::mbar_init(bar(C::BAR_MF + w * C::M_STAGES + st), 1);
                ptx::mbar_init(bar(C::BAR_ME + w * C::M_STAGES + st), 1 + 4);  // the MMA's commit + 4 softmax warps
            }
            for (int hf = 0; hf < 2; ++hf) {
                ptx::mbar_init(bar(C::BAR_SF + 2 * w + hf), 1);
                ptx::mbar_init(bar(C::BAR_PF + 2 * w + hf), 4);
            }
            ptx::mbar_init(bar(C::BAR_OA + w), 1);
            ptx::mbar_init(bar(C::BAR_PE + w), 1);
            ptx::mbar_init(bar(C::BAR_DRAIN + w), 1);
        }
        for (int st = 0; st < 2; ++st) {
            ptx::mbar_init(bar(C::BAR_BF + st), 1);
            ptx::mbar_init(bar(C::BAR_BE + st), 4 * C::NS);
        }
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 0) {
        // The A tile of the mask step: columns 0-2 = 1.0 (bf16), rest 0.  The
        // mask-column B tiles start zeroed; only columns 0-2 are rewritten.
        for (int c = lane; c < (C::AUG_TILE * (1 + C::NS * C::M_STAGES)) / 16; c += 32) {
            const uint32_t addr = (c < C::AUG_TILE / 16) ? sb + C::OFF_QAUG + uint32_t(c) * 16u
                                                         : sb + C::OFF_KAUG + uint32_t(c - C::AUG_TILE / 16) * 16u;
            ptx::st_shared_v4(addr, make_uint4(0u, 0u, 0u, 0u));
        }
        __syncwarp();
        for (int r = lane; r < kBM; r += 32)
            ptx::st_shared_v2(sb + C::OFF_QAUG + swz_chunk<C::AUG_ROW>(r, 0), 0x3F803F80u, 0x00003F80u);
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
    // The register hand-over (setmaxnreg) sits at the top of each role's
    // branch, so that the compiler sees which budget the role's code runs under.
    if (warp < 4) {
        if constexpr (C::SPLIT_REGS) ptx::setmaxnreg_dec<C::HELPER_REGS>();
        if (warp == 0) {
            // ------------------------------------------ bias tiles and masks
            // The bias tile of every (tile, block), shared by the three
            // slices, and the mask columns of every (tile, block, slice):
            // the block's 128 mask values relative to c = the slice's running
            // mask maximum (an online max over blocks), c to the softmax
            // through mc_s.  The mask values of the next block are fetched
            // from global memory before this block's are written, so their
            // latency overlaps a block.
            const bool bias_tma = HAS_PAIR && p.pair_g == nullptr;
            if (bias_tma && lane == 0) ptx::prefetch_tmap(&tm_pair);
            int b_issued = 0, m_done[C::NS] = {};
            float c_run[C::NS];
#pragma unroll
            for (int w = 0; w < C::NS; ++w) c_run[w] = -INFINITY;
            uint32_t raw[C::NS][4];
            auto fetch = [&](int L, int j) {
                const TriTile t = tri_tile(p, L, C::NS);
#pragma unroll
                for (int w = 0; w < C::NS; ++w) {
                    const uint16_t* mrow = (p.mask != nullptr && w < t.nv)
                                               ? p.mask + (size_t(t.b) * p.N + t.n0 + w) * size_t(p.S)
                                               : nullptr;
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int key = j * kBN + lane + 32 * k;
                        raw[w][k] = (mrow != nullptr && key < p.S) ? uint32_t(__ldg(mrow + key)) : 0u;
                    }
                }
            };
            bool ok = true;
            if (aug) fetch(first_tile, 0);
            for (int it = 0, L = first_tile; L < p.num_tiles && ok; ++it, L += G) {
                const TriTile t = tri_tile(p, L, C::NS);
                for (int j = 0; j < nkb && ok; ++j) {
                    if (bias_tma) {
                        const int st = b_issued % C::B_RING;
                        ok = wait_warp(bar(C::BAR_BE + st), ((b_issued / C::B_RING) & 1) ^ 1, abort_flag);
                        if (!ok) break;
                        if (lane == 0) {
                            const uint32_t dst = sb + C::OFF_BIAS + st * C::BIAS_BYTES;
                            ptx::mbar_arrive_expect_tx(bar(C::BAR_BF + st), C::BIAS_BYTES);
                            ptx::tma_load_3d(dst, &tm_pair, bar(C::BAR_BF + st), j * kBN, t.qb * kBM, t.b * p.H + t.h);
                            ptx::tma_load_3d(dst + C::BIAS_BYTES / 2, &tm_pair, bar(C::BAR_BF + st), j * kBN + 64,
                                             t.qb * kBM, t.b * p.H + t.h);
                        }
                        __syncwarp();
                        ++b_issued;
                    }
                    if (!aug) continue;
                    uint32_t cur[C::NS][4];
#pragma unroll
                    for (int w = 0; w < C::NS; ++w)
#pragma unroll
                        for (int k = 0; k < 4; ++k) cur[w][k] = raw[w][k];
                    if (j + 1 < nkb) fetch(L, j + 1);
                    else if (L + G < p.num_tiles) fetch(L + G, 0);
#pragma unroll
                    for (int w = 0; w < C::NS; ++w) {
                        if (!ok || w >= t.nv) break;
                        if (j == 0) c_run[w] = -INFINITY;
                        float v[4];
                        float bmax = -INFINITY;
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const int key = j * kBN + lane + 32 * k;
                            v[k] = key < p.S ? elem_to_f32<F16>(cur[w][k]) : -INFINITY;
                            bmax = fmaxf(bmax, v[k]);
                        }
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, o));
                        c_run[w] = fmaxf(c_run[w], bmax);
                        const float csub = (c_run[w] == -INFINITY) ? 0.f : c_run[w];
                        const int ms = w * C::M_STAGES + m_done[w] % C::M_STAGES;
                        ok = wait_warp(bar(C::BAR_ME + ms), ((m_done[w] / C::M_STAGES) & 1) ^ 1, abort_flag);
                        if (!ok) break;
                        const uint32_t tile = sb + C::OFF_KAUG + uint32_t(ms * C::AUG_TILE);
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const int key = lane + 32 * k;
                            // (mask - c) * sqrt(D) as hi + mid + lo, three bf16 that sum to the fp32 value.
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
                        ++m_done[w];
                    }
                }
            }
            if (!ok && bias_tma && lane == 0) {
                // Let every bias copy this warp started land before the CTA exits.
                for (int i2 = (b_issued > C::B_RING ? b_issued - C::B_RING : 0); i2 < b_issued; ++i2)
                    wait_bounded(bar(C::BAR_BF + i2 % C::B_RING), (i2 / C::B_RING) & 1, nullptr);
            }
            __syncwarp();
        } else if (warp - 1 < C::NS) {
            // ------------------------------------------- helper of slice w
            // Warp 1 + w drives slice n0 + w through every tile that has it:
            // its Q, K and V loads, the conversion of its V tiles to fp16, and
            // its MMAs, issued by one elected lane of the converged warp.  Per
            // block n of the slice's stream of (tile, key block) positions:
            //   load V(n+1) into the stage P.V(n-1) has released;
            //   wait until the softmax has written P(n); issue P.V(n);
            //   issue Q K^T(n+1) into the same columns (it runs after P.V(n));
            //   load K(n+2) into the stage Q K^T(n) has released (P(n) is
            //   written, so the softmax saw S(n), so Q K^T(n) is complete),
            //   and Q of the next tile once the last Q K^T of this one is done;
            //   convert V(n+1).
            const int w = warp - 1;
            // the slice's stream: position = (tile index L, key block j)
            auto first_pos = [&](int L, int& outL) -> bool {
                for (; L < p.num_tiles; L += G)
                    if (w < tri_tile(p, L, C::NS).nv) { outL = L; return true; }
                return false;
            };
            auto next_pos = [&](int L, int j, int& nL, int& nj) -> bool {
                if (j + 1 < nkb) { nL = L; nj = j + 1; return true; }
                nj = 0;
                return first_pos(L + G, nL);
            };
            auto coords = [&](int L, int& h, int& q0, int& bn) {
                const TriTile t = tri_tile(p, L, C::NS);
                h = t.h;
                q0 = t.qb * kBM;
                bn = t.b * p.N + t.n0 + w;
            };
            auto q_tile = [&](int qb) -> uint32_t { return sb + C::OFF_Q + uint32_t((w * C::Q_BUFS + qb) * C::TILE); };
            const uint64_t a_aug = desc_k_major<C::AUG_ROW>(sb + C::OFF_QAUG);
            const uint32_t d_s = tmem + C::TM_S0 + 128u * w;
            const uint32_t d_o = tmem + C::TM_O0 + uint32_t(D) * w;
            auto k_tile = [&](int st) -> uint32_t { return sb + C::OFF_K + uint32_t((w * C::K_STAGES + st) * C::TILE); };
            auto v_tile = [&](int st) -> uint32_t { return sb + C::OFF_V + uint32_t((w * C::V_STAGES + st) * C::TILE); };
            // one tile = NSUB boxes of SUBW elements per row, one barrier
            auto load_tile = [&](uint32_t dst, const CUtensorMap* m, uint32_t bar_addr, int h, int row0, int bn) {
                ptx::tma_load_4d_elect(dst, m, bar_addr, uint32_t(C::TILE), 0, h, row0, bn);
#pragma unroll
                for (int sub = 1; sub < C::NSUB; ++sub)
                    ptx::tma_load_4d_more_elect(dst + uint32_t(sub * C::SUBTILE), m, bar_addr, sub * C::SUBW, h, row0, bn);
            };
            auto load_k = [&](int n, int L, int j) {
                int h, q0, bn;
                coords(L, h, q0, bn);
                const int st = n % C::K_STAGES;
                load_tile(k_tile(st), &tm_k, bar(C::BAR_KF + w * C::K_STAGES + st), h, j * kBN, bn);
            };
            auto load_v = [&](int n, int L, int j) {
                int h, q0, bn;
                coords(L, h, q0, bn);
                const int st = n % C::V_STAGES;
                load_tile(v_tile(st), &tm_v, bar(C::BAR_VF + w * C::V_STAGES + st), h, j * kBN, bn);
            };
            // Q of the slice's tile number tq (its buffer tq % Q_BUFS)
            auto load_q = [&](int L, int tq) {
                int h, q0, bn;
                coords(L, h, q0, bn);
                const int qb = tq % C::Q_BUFS;
                load_tile(q_tile(qb), &tm_q, bar(C::BAR_QF + w * C::Q_BUFS + qb), h, q0, bn);
            };
            int n = 0, q_loads = 0, k_loads = 0, v_loads = 0;
            int tcur = 0;  // the slice's tile number of stream position n
            bool issued_any = false;
            // Q K^T of stream position n (block j of its tile) for keys 64 hf ..
            // 64 hf + 63, into S columns 64 hf ..; the first half waits for K(n),
            // the mask columns and (first block of a tile) Q
            auto issue_qk = [&](int nn, int j, int hf, int tq) -> bool {
                const int st = nn % C::K_STAGES;
                const int ms = w * C::M_STAGES + nn % C::M_STAGES;
                const int qb = tq % C::Q_BUFS;
                const uint64_t a_q = desc_k_major<C::ROW>(q_tile(qb));
                if (hf == 0) {
                    if (j == 0 && !wait_warp(bar(C::BAR_QF + w * C::Q_BUFS + qb), (tq / C::Q_BUFS) & 1, abort_flag))
                        return false;
                    if (!wait_warp(bar(C::BAR_KF + w * C::K_STAGES + st), (nn / C::K_STAGES) & 1, abort_flag))
                        return false;
                    if (aug && !wait_warp(bar(C::BAR_MF + ms), (nn / C::M_STAGES) & 1, abort_flag)) return false;
                    ptx::tc_fence_after();
                }
                const uint64_t bd = desc_k_major<C::ROW>(k_tile(st) + uint32_t(hf * 64 * C::ROW));
                const uint32_t d = d_s + 64u * hf;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    // K step kk: 32 B into its sub-tile's swizzled rows (descriptor units of 16 B)
                    const uint64_t off = uint64_t((kk / C::KPA) * (C::SUBTILE >> 4) + 2 * (kk % C::KPA));
                    ptx::mma_ss_elect(d, a_q + off, bd + off, C::IDESC_QK, kk > 0 ? 1u : 0u);
                }
                if (aug)
                    ptx::mma_ss_elect(d, a_aug,
                                      desc_k_major<C::AUG_ROW>(sb + C::OFF_KAUG + ms * C::AUG_TILE + hf * 64 * C::AUG_ROW),
                                      C::IDESC_MASK, 1u);
                if (hf == 1) {
                    if (aug) ptx::mma_commit_elect(bar(C::BAR_ME + ms));
                    ptx::mma_commit_elect(bar(C::BAR_KE + w * C::K_STAGES + st));
                }
                ptx::mma_commit_elect(bar(C::BAR_SF + 2 * w + hf));
                issued_any = true;
                return true;
            };
            // P.V of keys 64 hf .. 64 hf + 63 of stream position n
            auto issue_pv = [&](int nn, int j, int hf) {
                const int st = nn % C::V_STAGES;
                // V as the MN-major B operand: N = D in NSUB atoms SUBTILE bytes apart
                const uint64_t bd = desc_mn_major<C::ROW>(v_tile(st), uint32_t(C::SUBTILE));
#pragma unroll
                for (int kk = 0; kk < kBN / 32; ++kk) {  // 16 keys per K step = 16 rows of V
                    // keys 64 hf + 16 kk .. +15: P in columns 64 hf + 8 kk .. (fp16 pairs), V rows key0 ..
                    const int key0 = 64 * hf + 16 * kk;
                    ptx::mma_ts_elect(d_o, d_s + uint32_t(64 * hf + 8 * kk), bd + uint64_t((key0 * C::ROW) >> 4),
                                      C::IDESC_PV, (j > 0 || hf > 0 || kk > 0) ? 1u : 0u);
                }
            };
            int L = 0, j = 0;
            bool ok = first_pos(first_tile, L);
            const bool has_work = ok;
            if (ok) {
                if (lane == 0) {
                    ptx::prefetch_tmap(&tm_q);
                    ptx::prefetch_tmap(&tm_k);
                    ptx::prefetch_tmap(&tm_v);
                }
                __syncwarp();
                load_q(L, 0);
                ++q_loads;
                load_k(0, L, 0);
                ++k_loads;
                int L1, j1;
                if (next_pos(L, 0, L1, j1)) {
                    load_k(1, L1, j1);
                    ++k_loads;
                }
                load_v(0, L, 0);
                ++v_loads;
                ok = wait_warp(bar(C::BAR_VF + w * C::V_STAGES), 0, abort_flag);
                if (ok && !F16) convert_v_chunks<0, C::V_CHUNKS, true>(v_tile(0), lane);
                ok = ok && issue_qk(0, 0, 0, 0) && issue_qk(0, 0, 1, 0);
                if (ok && C::Q_BUFS == 1 && next_pos(L, 0, L1, j1) && j1 == 0) {
                    // one key block per tile and one Q buffer: position 1 needs the
                    // next Q as soon as Q K^T(0) is done
                    ok = wait_warp(bar(C::BAR_KE + w * C::K_STAGES), 0, abort_flag);
                    if (ok) {
                        load_q(L1, 1);
                        ++q_loads;
                    }
                }
            }
            while (ok) {
                int L1 = 0, j1 = 0, L2 = 0, j2 = 0;
                const bool has1 = next_pos(L, j, L1, j1);
                const bool has2 = has1 && next_pos(L1, j1, L2, j2);
                // V(n+1) into the stage of V(n-1), once P.V(n-1) is done (with one
                // stage, after P.V(n) below)
                if (C::V_STAGES >= 2 && has1) {
                    const int st = (n + 1) % C::V_STAGES;
                    if (n >= 1) ok = wait_warp(bar(C::BAR_VE + w * C::V_STAGES + st), ((n - 1) / C::V_STAGES) & 1, abort_flag);
                    if (!ok) break;
                    load_v(n + 1, L1, j1);
                    ++v_loads;
                }
                const int tnext = (has1 && j1 == 0) ? tcur + 1 : tcur;  // tile number of position n+1
                // keys 0-63 of block n: P.V, then Q K^T of keys 0-63 of block n+1
                ok = wait_warp(bar(C::BAR_PF + 2 * w), n & 1, abort_flag);
                if (!ok) break;
                ptx::tc_fence_after();
                issue_pv(n, j, 0);
                ptx::mma_commit_elect(bar(C::BAR_OA + w));
                if (C::Q_BUFS >= 2 && j == 0) {
                    // First block of a tile: every Q K^T of the previous tile is
                    // complete (the softmax has seen S(n)), so its Q buffer takes
                    // the next tile's Q, which then lands during this tile.
                    int Ln;
                    if (first_pos(L + G, Ln)) {
                        load_q(Ln, tcur + 1);
                        ++q_loads;
                    }
                }
                if (has1 && !issue_qk(n + 1, j1, 0, tnext)) { ok = false; break; }
                // keys 64-127 of block n: P.V, then Q K^T of keys 64-127 of block n+1
                ok = wait_warp(bar(C::BAR_PF + 2 * w + 1), n & 1, abort_flag);
                if (!ok) break;
                ptx::tc_fence_after();
                issue_pv(n, j, 1);
                ptx::mma_commit_elect(bar(C::BAR_VE + w * C::V_STAGES + n % C::V_STAGES));
                if (j == nkb - 1) ptx::mma_commit_elect(bar(C::BAR_PE + w));
                if (!has1) break;
                if (!issue_qk(n + 1, j1, 1, tnext)) { ok = false; break; }
                if (C::V_STAGES == 1) {
                    ok = wait_warp(bar(C::BAR_VE + w), n & 1, abort_flag);
                    if (!ok) break;
                    load_v(n + 1, L1, j1);
                    ++v_loads;
                }
                // K(n+2) into the stage of K(n) (Q K^T(n) is complete: the softmax saw S(n))
                if (has2) {
                    load_k(n + 2, L2, j2);
                    ++k_loads;
                    if (C::Q_BUFS == 1 && j2 == 0) {
                        // one Q buffer: the next tile's Q once Q K^T(n+1), the last
                        // one of this tile, is done
                        const int st = (n + 1) % C::K_STAGES;
                        ok = wait_warp(bar(C::BAR_KE + w * C::K_STAGES + st), ((n + 1) / C::K_STAGES) & 1, abort_flag);
                        if (!ok) break;
                        load_q(L2, tnext + 1);
                        ++q_loads;
                    }
                }
                // V(n+1) to fp16
                {
                    const int st = (n + 1) % C::V_STAGES;
                    ok = wait_warp(bar(C::BAR_VF + w * C::V_STAGES + st), ((n + 1) / C::V_STAGES) & 1, abort_flag);
                    if (!ok) break;
                    if (!F16) convert_v_chunks<0, C::V_CHUNKS, true>(v_tile(st), lane);
                }
                L = L1;
                j = j1;
                tcur = tnext;
                ++n;
            }
            if (!ok && has_work) {
                // Every MMA and copy this warp started completes before the CTA
                // frees tensor memory and exits.
                if (issued_any) {
                    ptx::mma_commit_elect(bar(C::BAR_DRAIN + w));
                    wait_warp(bar(C::BAR_DRAIN + w), 0, nullptr);
                }
                if (lane == 0) {
                    for (int i2 = (q_loads > C::Q_BUFS ? q_loads - C::Q_BUFS : 0); i2 < q_loads; ++i2)
                        wait_bounded(bar(C::BAR_QF + w * C::Q_BUFS + i2 % C::Q_BUFS), (i2 / C::Q_BUFS) & 1, nullptr);
                    for (int i2 = (k_loads > C::K_STAGES ? k_loads - C::K_STAGES : 0); i2 < k_loads; ++i2)
                        wait_bounded(bar(C::BAR_KF + w * C::K_STAGES + i2 % C::K_STAGES), (i2 / C::K_STAGES) & 1, nullptr);
                    for (int i2 = (v_loads > C::V_STAGES ? v_loads - C::V_STAGES : 0); i2 < v_loads; ++i2)
                        wait_bounded(bar(C::BAR_VF + w * C::V_STAGES + i2 % C::V_STAGES), (i2 / C::V_STAGES) & 1, nullptr);
                }
            }
            __syncwarp();
        }
    } else {
        // ------------------------------------------------------------ softmax
        if constexpr (C::SPLIT_REGS) ptx::setmaxnreg_inc<C::SOFTMAX_REGS>();
        const int w = (warp - 4) >> 2;   // slice (n0 + w)
        const int quarter = warp & 3;    // TMEM lanes 32*quarter .. +31
        const int r = quarter * 32 + lane;
        const uint32_t lane_base = uint32_t(quarter * 32) << 16;
        const uint32_t tS = tmem + lane_base + C::TM_S0 + 128u * w;
        const uint32_t tO = tmem + lane_base + C::TM_O0 + uint32_t(D) * w;
        const float2 sqd2 = make_float2(p.sqrt_d, p.sqrt_d);
        const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
        const float inv_c = 1.0f / p.scale_log2;
        const bool bias_tma = HAS_PAIR && p.pair_g == nullptr;
        int blk = 0;     // blocks of this slice processed (phase of SF / PF)
        int tiles = 0;   // tiles of this slice finished (phase of PE)
        int b_seen = 0;  // bias tiles consumed (every tile, valid slice or not)
        int m_seen = 0;  // mask stages of this slice consumed
        bool ok = true;
        for (int it = 0, L = first_tile; L < p.num_tiles && ok; ++it, L += G) {
            const TriTile t = tri_tile(p, L, C::NS);
            if (w >= t.nv) {
                // No slice n0 + w in this tile: only release the shared bias tiles.
                if (bias_tma)
                    for (int j = 0; j < nkb && ok; ++j, ++b_seen) {
                        const int bs = b_seen % C::B_RING;
                        ok = wait_warp(bar(C::BAR_BF + bs), (b_seen / C::B_RING) & 1, abort_flag);
                        if (ok) ptx::mbar_arrive_elect(bar(C::BAR_BE + bs));
                    }
                continue;
            }
            float m = -INFINITY;   // running maximum (log2 units, relative to the rebase c_cur)
            float thr = -INFINITY; // raw-score threshold (m + 12) / (log2(e) / sqrt(D))
            float c_cur = 0.f;     // mask rebase that m and the stored P are relative to
            float2 suma = make_float2(0.f, 0.f), sumb = make_float2(0.f, 0.f);
            for (int j = 0; j < nkb && ok; ++j, ++blk) {
                // S of keys 0-63 (keys 64-127 are waited for at step 2)
                ok = wait_warp(bar(C::BAR_SF + 2 * w), blk & 1, abort_flag);
                if (!ok) break;
                ptx::tc_fence_after();
                bool half_b_ready = false;  // S of keys 64-127 of this block waited for
                // Waits for S of keys 64-127: after it, P.V of keys 64-127 of the
                // previous block (issued just before that Q K^T) is complete.
                auto wait_half_b = [&]() -> bool {
                    if (half_b_ready) return true;
                    if (!wait_warp(bar(C::BAR_SF + 2 * w + 1), blk & 1, abort_flag)) return false;
                    ptx::tc_fence_after();
                    half_b_ready = true;
                    return true;
                };
                float s[32];  // one 32-key step of S(j), then t in place
                if (aug) {
                    const int ms = w * C::M_STAGES + m_seen % C::M_STAGES;
                    ok = wait_warp(bar(C::BAR_MF + ms), (m_seen / C::M_STAGES) & 1, abort_flag);
                    if (!ok) break;
                    const float cs = mc_s[ms];
                    ptx::mbar_arrive_elect(bar(C::BAR_ME + ms));
                    ++m_seen;
                    if (cs != c_cur) {
                        // the rebase grew: earlier logits are relative to a smaller c
                        m -= (cs - c_cur) * kLog2e;
                        thr = (m + kTriRescaleThreshold) * inv_c;
                        c_cur = cs;
                    }
                }
                const int bs = b_seen % C::B_RING;
                uint32_t brow = 0;
                if (bias_tma) {
                    ok = wait_warp(bar(C::BAR_BF + bs), (b_seen / C::B_RING) & 1, abort_flag);
                    if (!ok) break;
                    brow = (sb + C::OFF_BIAS + uint32_t(bs * C::BIAS_BYTES) + uint32_t(r * 128)) |
                           uint32_t((r & 7) << 4);
                    ++b_seen;
                }
                // bias words of a step (keys 32c .. 32c+31: 16 B groups 4c .. 4c+3 of the row)
                // the row of pair bias this thread reads from global memory
                // (S % 8 != 0); beyond S it reads nothing and adds 0 (those
                // keys are -inf through the mask columns, those rows unused)
                const uint16_t* grow = (HAS_PAIR && !bias_tma && t.qb * kBM + r < p.S)
                                           ? p.pair_g + (size_t(t.b * p.H + t.h) * p.S + size_t(t.qb * kBM + r)) * p.S
                                           : nullptr;
                auto load_bias = [&](int c, uint4* bw) {
                    if (HAS_PAIR) {
                        if (bias_tma) {
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                const int g = 4 * c + q;
                                bw[q] = ptx::ld_shared_v4((brow ^ uint32_t((g & 7) << 4)) +
                                                          uint32_t((g >> 3) * (C::BIAS_BYTES / 2)));
                            }
                        } else {
                            uint32_t wds[16];
#pragma unroll
                            for (int e = 0; e < 16; ++e) {
                                const int key = j * kBN + 32 * c + 2 * e;
                                const uint32_t lo = (grow != nullptr && key < p.S) ? uint32_t(__ldg(grow + key)) : 0u;
                                const uint32_t hi =
                                    (grow != nullptr && key + 1 < p.S) ? uint32_t(__ldg(grow + key + 1)) : 0u;
                                wds[e] = lo | (hi << 16);
                            }
#pragma unroll
                            for (int q = 0; q < 4; ++q)
                                bw[q] = make_uint4(wds[4 * q], wds[4 * q + 1], wds[4 * q + 2], wds[4 * q + 3]);
                        }
                    }
                };
                // One 32-key step per trip of a loop that is not unrolled: the
                // body, with its rare path, stays small enough for the
                // instruction cache that the softmax warpgroups and the helpers
                // share.
                // P of step c goes to columns 16 c (keys 0-63) or 64 + 16 (c - 2)
                // (keys 64-127): each over scores of its own half already read,
                // so that Q K^T of keys 0-63 of the next block may overwrite
                // columns 0-63 while the P of keys 64-127 waits for its P.V.
                auto pcol = [](int c) -> uint32_t { return uint32_t(c < 2 ? 16 * c : 64 + 16 * (c - 2)); };
                // S and the bias words of step c + 1 are requested as soon as step
                // c no longer needs its registers (after its exps and its check),
                // so their latency overlaps the stores of step c.
                // Without a pair bias the S of step c + 1 is requested as soon as
                // step c no longer needs its registers (after its exps and its
                // check), so its latency overlaps the stores of step c.  With a
                // pair bias, S and the bias words are requested at the top of
                // each step (measured faster there).
                constexpr bool kEarlyS = !HAS_PAIR;
                if (kEarlyS) tmem_ld_x32f(tS, s);
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint4 bw[4];
                    if (!kEarlyS) tmem_ld_x32f(tS + 32u * c, s);
                    load_bias(c, bw);
                    tmem_wait_x32f(s);
                    // One basic block per step: t = S + pair * sqrt(D) and
                    // p = 2^(t log2(e) / sqrt(D) - m) against the current m, all
                    // independent per key pair, so the exp unit is fed while the
                    // adds proceed.  The check that m still covers the step comes
                    // after; when it does not (rare), the step is recomputed from
                    // t (kept in s).
                    float2 csa = make_float2(0.f, 0.f), csb = make_float2(0.f, 0.f);
                    uint32_t pk[16];
                    {
                        const float m_safe = (m == -INFINITY) ? 0.f : m;  // an all -inf row keeps p = 0
                        const float2 nm2 = make_float2(-m_safe, -m_safe);
                        auto step_pair = [&](int e, uint32_t bwd) {
                            const int k = 2 * e;
                            float2 tt;
                            const float2 sv = make_float2(s[k], s[k + 1]);
                            if (!HAS_PAIR) tt = sv;
                            else if constexpr (F16) tt = __ffma2_rn(pair_to_f32x2<F16>(bwd), sqd2, sv);
                            else tt = bf16x2_fma2(bwd, sqd2, sv);
                            s[k] = tt.x;
                            s[k + 1] = tt.y;
                            const float2 x = __ffma2_rn(tt, sc2, nm2);
                            const float p0 = ptx::ex2_approx(x.x);
                            const float p1 = ptx::ex2_approx(x.y);
                            if (e & 1) csb = __fadd2_rn(csb, make_float2(p0, p1));
                            else csa = __fadd2_rn(csa, make_float2(p0, p1));
                            pk[e] = ptx::pack_f16x2(p0, p1);  // P column 16c + e: keys 32c + 2e (low), + 1
                        };
                        if (HAS_PAIR) {
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                const uint32_t wd[4] = {bw[q].x, bw[q].y, bw[q].z, bw[q].w};
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    step_pair(4 * q + e, wd[e]);
                                }
                            }
                            if (bias_tma && c == 3) ptx::mbar_arrive_elect(bar(C::BAR_BE + bs));
                        } else {
#pragma unroll
                            for (int e = 0; e < 16; ++e) step_pair(e, 0u);
                        }
                    }
                    // The step's p sum bounds each of its p: at most 2^15 means
                    // every p fits (the maximum is only needed when it does not,
                    // and at the first step of a tile, where m is still -inf).
                    const float2 cst = __fadd2_rn(csa, csb);
                    const bool check = (cst.x + cst.y > kStepSumLimit) || (m == -INFINITY);
                    if (__any_sync(0xffffffffu, check)) {
                        float mx = -INFINITY;
#pragma unroll
                        for (int e = 0; e < 32; e += 2) mx = max3f(mx, s[e], s[e + 1]);
                        const bool raise = mx > thr;
                        // Where the step exceeds the running maximum by more than
                        // 15 (always so for the first step of a tile): move m to
                        // the step maximum, rescale what is already accumulated
                        // relative to the old m, and recompute this step.
                        float alpha = 1.f;
                        if (raise) {
                            // Never a factor above 1: when the mask rebase has
                            // just jumped (a block after fully masked ones), m
                            // and a chunk of still-masked keys can both be near
                            // -1e9 log2(e), their fp32 difference noise; what is
                            // accumulated then is scaled to 0 by the raise of the
                            // block's first unmasked chunk.
                            const float m_new = mx * p.scale_log2;
                            alpha = ptx::ex2_approx(fminf(m - m_new, 0.f));  // 0 while m is -inf
                            m = m_new;
                            thr = (m + kTriRescaleThreshold) * inv_c;
                        }
                        suma = make_float2(suma.x * alpha, suma.y * alpha);
                        sumb = make_float2(sumb.x * alpha, sumb.y * alpha);
                        if (__any_sync(0xffffffffu, alpha != 1.f)) {
                            ptx::tmem_st_wait();
                            // P of this block's earlier steps that the tensor core
                            // has not taken yet (fp16, 16 columns per step)
#pragma unroll 1
                            for (int k = (c < 2 ? 0 : 2); k < c; ++k) {
                                uint32_t ok16[16];
                                ptx::tmem_ld_x16(tS + pcol(k), ok16);
                                ptx::tmem_ld_wait_x16(ok16);
#pragma unroll
                                for (int e = 0; e < 16; ++e) {
                                    const __half2 h2 = *reinterpret_cast<const __half2*>(&ok16[e]);
                                    const float2 f = __half22float2(h2);
                                    ok16[e] = ptx::pack_f16x2(f.x * alpha, f.y * alpha);
                                }
                                ptx::tmem_st_x16(tS + pcol(k), ok16);
                            }
                            // O holds the earlier blocks and, from step 2 on, P.V of
                            // keys 0-63 of this block; rescale it once the P.V
                            // writing it are done: in steps 0-1 the last one is
                            // keys 64-127 of the previous block, in steps 2-3 keys
                            // 0-63 of this one.  (In block 0 before step 2, O holds
                            // nothing yet: its first P.V overwrites it.)
                            if (j > 0 || c >= 2) {
                                bool ready = (c >= 2) ? wait_warp(bar(C::BAR_OA + w), blk & 1, abort_flag)
                                                      : wait_half_b();
                                if (!ready) { ok = false; break; }
                                ptx::tc_fence_after();
                                constexpr int OCH = D < 32 ? D : 32;  // O columns per load
#pragma unroll
                                for (int oc = 0; oc < D; oc += OCH) {
                                    uint32_t o[OCH];
                                    if constexpr (OCH == 32) {
                                        ptx::tmem_ld_x32(tO + oc, o);
                                        ptx::tmem_ld_wait_x32(o);
                                    } else {
                                        ptx::tmem_ld_x16(tO + oc, o);
                                        ptx::tmem_ld_wait_x16(o);
                                    }
#pragma unroll
                                    for (int e = 0; e < OCH; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
#pragma unroll
                                    for (int e = 0; e < OCH; e += 16) ptx::tmem_st_x16(tO + oc + e, o + e);
                                }
                            }
                        }
                        const float m_safe = (m == -INFINITY) ? 0.f : m;
                        const float2 nm2 = make_float2(-m_safe, -m_safe);
                        csa = make_float2(0.f, 0.f);
                        csb = make_float2(0.f, 0.f);
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            const float2 x = __ffma2_rn(make_float2(s[2 * e], s[2 * e + 1]), sc2, nm2);
                            const float p0 = ptx::ex2_approx(x.x);
                            const float p1 = ptx::ex2_approx(x.y);
                            if (e & 1) csb = __fadd2_rn(csb, make_float2(p0, p1));
                            else csa = __fadd2_rn(csa, make_float2(p0, p1));
                            pk[e] = ptx::pack_f16x2(p0, p1);
                        }
                    }
                    suma = __fadd2_rn(suma, csa);
                    sumb = __fadd2_rn(sumb, csb);
                    if (c == 1) {
                        // hand P of keys 0-63 to the tensor core, then wait for S of keys 64-127
                        ptx::tmem_st_x8(tS + pcol(c), pk);
                        ptx::tmem_st_x8(tS + pcol(c) + 8u, pk + 8);
                        ptx::tmem_st_wait();
                        ptx::tc_fence_before();
                        ptx::mbar_arrive_elect(bar(C::BAR_PF + 2 * w));
                        if (!(ok = wait_half_b())) break;
                    }
                    if (kEarlyS && c < 3) tmem_ld_x32f(tS + 32u * (c + 1), s);
                    if (c != 1) {
                        ptx::tmem_st_x8(tS + pcol(c), pk);
                        ptx::tmem_st_x8(tS + pcol(c) + 8u, pk + 8);
                    }
                }
                if (!ok) break;
                ptx::tmem_st_wait();
                ptx::tc_fence_before();
                ptx::mbar_arrive_elect(bar(C::BAR_PF + 2 * w + 1));
            }
            // -------------------------------------------------------- epilogue
            if (ok) ok = wait_warp(bar(C::BAR_PE + w), tiles & 1, abort_flag);
            ++tiles;
            if (!ok) break;
            ptx::tc_fence_after();
            const float l = (suma.x + suma.y) + (sumb.x + sumb.y);
            const int n = t.n0 + w;
            const int row = t.qb * kBM + r;
            {
                const float inv_l = l > 0.f ? 1.f / l : 0.f;
                bool finite = (l < INFINITY);  // an fp16 overflow of V shows up in O
                uint16_t* orow = p.out + ((size_t(t.b) * p.N + n) * size_t(p.S) + size_t(row)) * size_t(p.H) * D +
                                 size_t(t.h) * D;
                constexpr int OCH = D < 32 ? D : 32;  // O columns per load
                // the tensor-memory loads are warp-collective: every lane takes
                // them, only lanes with a row inside S store
#pragma unroll
                for (int oc = 0; oc < D; oc += OCH) {
                    uint32_t o[OCH];
                    if constexpr (OCH == 32) {
                        ptx::tmem_ld_x32(tO + oc, o);
                        ptx::tmem_ld_wait_x32(o);
                    } else {
                        ptx::tmem_ld_x16(tO + oc, o);
                        ptx::tmem_ld_wait_x16(o);
                    }
                    if (row < p.S) {
#pragma unroll
                        for (int k = 0; k < OCH; k += 8) {
                            float f[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                f[e] = __uint_as_float(o[k + e]) * inv_l;
                                finite = finite && fabsf(f[e]) < INFINITY;
                            }
                            uint4 v;
                            v.x = pack_out<F16>(f[0], f[1]);
                            v.y = pack_out<F16>(f[2], f[3]);
                            v.z = pack_out<F16>(f[4], f[5]);
                            v.w = pack_out<F16>(f[6], f[7]);
                            *reinterpret_cast<uint4*>(orow + oc + k) = v;
                        }
                    }
                }
                if (row < p.S) {
                    if (!finite) record_status(EVO_ERR_RANGE);
                    const float lse = l > 0.f ? (m + ptx::lg2_approx(l)) * kLn2 + c_cur : -INFINITY;
                    p.lse[((size_t(t.b) * p.N + n) * p.H + t.h) * size_t(p.S) + row] = lse;
                }
            }
        }
        // on an abort, no tensor-memory access of this thread may still be in
        // flight when the memory is freed
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        ptx::tmem_st_wait();
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {  // the warp that allocated
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace evo
