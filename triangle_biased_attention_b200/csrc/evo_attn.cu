// Host side of libevoattn.so: argument checks, TMA tensor-map encoding and
// kernel launch for the C ABI declared in include/evo_attn.h.
//
// The calling convention follows the DeepSpeed DS4Sci_EvoformerAttention
// guide's statement of the problem (hmyw.cn, section 5: one call for all four
// variants, Q/K/V in [*, L, Head, Dim], biases [B,N,1,1,S] and [B,1,H,S,S],
// a missing bias passed as "empty" -- here NULL -- through the same call, an
// fp32 log-sum-exp beside O), adapted to plain pointers and status codes: the
// guide's Python front end asserts on dtype and shapes, this library returns
// an evo_status_t before launching anything.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <type_traits>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "evo_attn.h"
#include "common.cuh"
#include "fwd_tri_sm100.cuh"
#include "fwd_f32.cuh"
#include "bwd_simt.cuh"
#include "bwd_tri_sm100.cuh"
#include "trimul_sm100.cuh"

namespace {


constexpr int kMaxDevices = 64;

// Sets a kernel's dynamic shared-memory limit once per device.  Calls from
// several host threads may race on the first use; a mutex orders them and
// the flag is only set once the attribute call has succeeded.
struct AttrOnce {
    std::mutex mu;
    bool done[kMaxDevices] = {};
    template <typename K>
    bool ensure(int dev, K kernel, int smem_bytes) {
        std::lock_guard<std::mutex> lock(mu);
        if (done[dev]) return true;
        if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes) != cudaSuccess)
            return false;
        done[dev] = true;
        return true;
    }
};

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

bool mul_ok(int64_t a, int64_t b, int64_t* out) { return !__builtin_mul_overflow(a, b, out); }

bool overlap(const void* a, int64_t abytes, const void* b, int64_t bbytes) {
    if (a == nullptr || b == nullptr || abytes <= 0 || bbytes <= 0) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + uint64_t(bbytes) && b0 < a0 + uint64_t(abytes);
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// The device that owns `ptr`, or a negative status if it is not device memory.
int device_of(const void* ptr) {
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, ptr) != cudaSuccess) {
        cudaGetLastError();
        return EVO_ERR_INVALID_ARG;
    }
    if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged) return EVO_ERR_INVALID_ARG;
    return attr.device;
}

// Makes the device that owns the buffers current for the duration of one
// call and restores the caller's current device afterwards.
struct DeviceScope {
    int prev = -1;
    bool changed = false;
    ~DeviceScope() {
        if (changed) cudaSetDevice(prev);
    }
};

// Relaxed stream-capture mode for this thread during one call, so that the
// call's host-side queries (pointer attributes, function attributes, the
// driver entry point) are allowed while the caller captures a CUDA graph;
// the launches and copies themselves are captured as usual.
struct RelaxedCapture {
    cudaStreamCaptureMode mode = cudaStreamCaptureModeRelaxed;
    RelaxedCapture() { cudaThreadExchangeStreamCaptureMode(&mode); }
    ~RelaxedCapture() { cudaThreadExchangeStreamCaptureMode(&mode); }
};

int select_device_of(const void* ptr, DeviceScope& scope) {
    const int dev = device_of(ptr);
    if (dev < 0) return dev;
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess) return EVO_ERR_CUDA;
    if (cur != dev) {
        if (cudaSetDevice(dev) != cudaSuccess) return EVO_ERR_CUDA;
        scope.prev = cur;
        scope.changed = true;
    }
    return dev;
}

// Q/K/V/O as a 4-D tensor {D, H, S, B*N}; a box is one (b, n, h) slice's
// 128 rows of `box_w` elements (D, or 64 for D = 128, whose rows are loaded as
// two boxes), swizzled over the box_w*2-byte row.
bool encode_qkv(CUtensorMap* m, const void* base, int64_t BN, int64_t S, int64_t H, int64_t D, int64_t box_w,
                CUtensorMapDataType dt) {
    const cuuint64_t dims[4] = {cuuint64_t(D), cuuint64_t(H), cuuint64_t(S), cuuint64_t(BN)};
    const cuuint64_t strides[3] = {cuuint64_t(D * 2), cuuint64_t(H * D * 2), cuuint64_t(S * H * D * 2)};
    const cuuint32_t box[4] = {cuuint32_t(box_w), 1, cuuint32_t(evo::kBM), 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUtensorMapSwizzle sw = box_w == 64 ? CU_TENSOR_MAP_SWIZZLE_128B
                                              : (box_w == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
    return encode_fn()(m, dt, 4, const_cast<void*>(base), dims, strides, box, estr,
                       CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Pair bias as a 3-D tensor {S (key j), S (query i), B*H}; a box is 128
// queries x 64 keys (128 B rows, 128 B swizzle).
bool encode_pair(CUtensorMap* m, const void* base, int64_t BH, int64_t S, CUtensorMapDataType dt) {
    const cuuint64_t dims[3] = {cuuint64_t(S), cuuint64_t(S), cuuint64_t(BH)};
    const cuuint64_t strides[2] = {cuuint64_t(S * 2), cuuint64_t(S * S * 2)};
    const cuuint32_t box[3] = {64, cuuint32_t(evo::kBM), 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return encode_fn()(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
                       CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The tcgen05 kernel: one CTA per SM, each walking the tiles (query block,
// head, group of n slices, batch) with a stride of the grid size.
template <int D, bool HAS_PAIR, bool F16>
int launch_tri(int dev, const void* Q, const void* K, const void* V, const void* mask, const void* pair, void* O,
               float* LSE, int64_t B, int64_t N, int64_t S, int64_t H, cudaStream_t stream) {
    using C = evo::TriCfg<D, HAS_PAIR, F16>;
    auto kernel = evo::evo_fwd_tri_kernel<D, HAS_PAIR, F16>;
    const CUtensorMapDataType dt = F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    static AttrOnce attr;
    if (!attr.ensure(dev, kernel, C::SMEM_BYTES)) return EVO_ERR_CUDA;
    if (C::SPLIT_REGS) {
        // the register hand-over (setmaxnreg) needs the whole split at launch
        cudaFuncAttributes fa;
        if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess ||
            fa.numRegs * C::THREADS < 128 * C::HELPER_REGS + C::NS * 128 * C::SOFTMAX_REGS)
            return EVO_ERR_CUDA;
    }
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
        return EVO_ERR_CUDA;
    CUtensorMap tq, tk, tv, tp;
    std::memset(&tp, 0, sizeof(tp));
    if (!encode_qkv(&tq, Q, B * N, S, H, D, C::SUBW, dt) || !encode_qkv(&tk, K, B * N, S, H, D, C::SUBW, dt) ||
        !encode_qkv(&tv, V, B * N, S, H, D, C::SUBW, dt))
        return EVO_ERR_CUDA;
    // a pair bias whose rows are whole 16-byte units comes through the TMA
    // ring; otherwise the softmax threads read it from global memory
    const bool pair_tma = HAS_PAIR && S % 8 == 0;
    if (pair_tma && !encode_pair(&tp, pair, B * H, S, dt)) return EVO_ERR_CUDA;

    evo::TriParams p;
    p.mask = static_cast<const uint16_t*>(mask);
    p.pair_g = (HAS_PAIR && !pair_tma) ? static_cast<const uint16_t*>(pair) : nullptr;
    p.out = static_cast<uint16_t*>(O);
    p.lse = LSE;
    p.N = int(N);
    p.S = int(S);
    p.H = int(H);
    p.num_kb = int((S + evo::kBN - 1) / evo::kBN);
    p.num_qb = int((S + evo::kBM - 1) / evo::kBM);
    p.num_ng = int((N + C::NS - 1) / C::NS);
    p.num_tiles = int(int64_t(p.num_qb) * H * p.num_ng * B);
    p.scale_log2 = float(1.4426950408889634 / std::sqrt(double(D)));
    p.sqrt_d = float(std::sqrt(double(D)));
    // the mask (or -inf for keys past S in a ragged last block) enters the score MMA
    p.aug = (mask != nullptr || S % evo::kBN != 0) ? 1 : 0;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(p.num_tiles < sms ? p.num_tiles : sms), 1, 1);
    cfg.blockDim = dim3(C::THREADS, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    return cudaLaunchKernelEx(&cfg, kernel, tq, tk, tv, tp, p) == cudaSuccess ? EVO_OK : EVO_ERR_CUDA;
}

// The SIMT kernel: T = float for fp32 inputs, uint16_t (bf16 bits) for the
// bf16 shapes the tensor-core kernel does not take.
template <typename T>
int launch_f32(int dev, const void* Q, const void* K, const void* V, const void* mask, const void* pair, void* O,
               float* LSE, int64_t B, int64_t N, int64_t S, int64_t H, int64_t D, cudaStream_t stream) {
    evo::F32Params<T> p;
    p.q = static_cast<const T*>(Q);
    p.k = static_cast<const T*>(K);
    p.v = static_cast<const T*>(V);
    p.mask = static_cast<const T*>(mask);
    p.pair = static_cast<const T*>(pair);
    p.out = static_cast<T*>(O);
    p.lse = LSE;
    p.N = int(N);
    p.S = int(S);
    p.H = int(H);
    p.D = int(D);
    p.ld = int(D) + 1;
    p.num_qb = int((S + evo::kF32Rows - 1) / evo::kF32Rows);
    p.scale = float(1.0 / std::sqrt(double(D)));
    const size_t smem = sizeof(float) * (size_t(2 * evo::kF32Keys + evo::kF32Rows) * p.ld +
                                         size_t(evo::kF32Rows) * evo::kF32Keys + evo::kF32Rows);
    static AttrOnce attr;
    const int max_smem = int(sizeof(float) * (size_t(2 * evo::kF32Keys + evo::kF32Rows) * (evo::kF32MaxD + 1) +
                                              size_t(evo::kF32Rows) * evo::kF32Keys + evo::kF32Rows));
    if (!attr.ensure(dev, evo::evo_fwd_f32_kernel<T>, max_smem)) return EVO_ERR_CUDA;
    const long long blocks = (long long)B * N * H * p.num_qb;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(blocks), 1, 1);
    cfg.blockDim = dim3(evo::kF32Rows * 32, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    return cudaLaunchKernelEx(&cfg, evo::evo_fwd_f32_kernel<T>, p) == cudaSuccess ? EVO_OK : EVO_ERR_CUDA;
}

// One warp initialises an mbarrier that expects one arrival, never arrives,
// and waits on it with a short limit: the wait must give up, record
// EVO_ERR_TIMEOUT and let the kernel finish.
__global__ void selftest_timeout_kernel(uint64_t limit_ns, int* result) {
    __shared__ __align__(8) uint64_t mbar;
    const uint32_t bar = evo::ptx::smem_u32(&mbar);
    if (threadIdx.x == 0) {
        evo::ptx::mbar_init(bar, 1);
        evo::ptx::fence_mbar_init();
    }
    __syncwarp();
    const bool ok = evo::wait_bounded_for(bar, 0, limit_ns);
    if (threadIdx.x == 0) *result = ok ? 1 : 0;
}

}  // namespace

extern "C" EVO_API int evo_attn_selftest_timeout(int64_t limit_ns, int* result, evo_stream_t stream) {
    if (limit_ns <= 0 || limit_ns > 1000000000ll || result == nullptr) return EVO_ERR_INVALID_ARG;
    DeviceScope scope;
    const int dev = select_device_of(result, scope);
    if (dev < 0) return dev;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1, 1, 1);
    cfg.blockDim = dim3(32, 1, 1);
    cfg.stream = reinterpret_cast<cudaStream_t>(stream);
    return cudaLaunchKernelEx(&cfg, selftest_timeout_kernel, uint64_t(limit_ns), result) == cudaSuccess
               ? EVO_OK
               : EVO_ERR_CUDA;
}

namespace {

// Every argument check of evo_attn_fwd that needs no CUDA call, in the order
// the header lists them.  On success *tensor_core says which kernel runs.
int check_fwd(const void* Q, const void* K, const void* V, const void* mask_bias, const void* pair_bias, void* O,
              float* LSE, int64_t B, int64_t N, int64_t S, int64_t H, int64_t D, int dtype, bool* tensor_core) {
    if (B < 0 || N < 0 || S < 0 || H < 0 || D < 0) return EVO_ERR_INVALID_ARG;
    if (dtype != EVO_DTYPE_BF16 && dtype != EVO_DTYPE_FP32 && dtype != EVO_DTYPE_FP16) return EVO_ERR_UNSUPPORTED_DTYPE;
    if (D == 0) return EVO_ERR_UNSUPPORTED_SHAPE;
    if (B == 0 || N == 0 || S == 0 || H == 0) return EVO_OK;  // nothing to compute
    if (!Q || !K || !V || !O || !LSE) return EVO_ERR_INVALID_ARG;

    const int64_t es = dtype == EVO_DTYPE_FP32 ? 4 : 2;
    int64_t bn, bns, bnsh, qkv_elems, qkv_bytes, mask_bytes, bh, pair_elems, pair_bytes, lse_bytes;
    if (!mul_ok(B, N, &bn) || !mul_ok(bn, S, &bns) || !mul_ok(bns, H, &bnsh) || !mul_ok(bnsh, D, &qkv_elems) ||
        !mul_ok(qkv_elems, es, &qkv_bytes) || !mul_ok(bns, es, &mask_bytes) || !mul_ok(B, H, &bh) ||
        !mul_ok(bh, S, &pair_elems) || !mul_ok(pair_elems, S, &pair_elems) ||
        !mul_ok(pair_elems, es, &pair_bytes) || !mul_ok(bnsh, 4, &lse_bytes))
        return EVO_ERR_UNSUPPORTED_SHAPE;

    // outputs must not overlap each other or any input
    const void* ins[5] = {Q, K, V, mask_bias, pair_bias};
    const int64_t in_bytes[5] = {qkv_bytes, qkv_bytes, qkv_bytes, mask_bytes, pair_bytes};
    if (overlap(O, qkv_bytes, LSE, lse_bytes)) return EVO_ERR_INVALID_ARG;
    for (int i = 0; i < 5; ++i)
        if (overlap(O, qkv_bytes, ins[i], in_bytes[i]) || overlap(LSE, lse_bytes, ins[i], in_bytes[i]))
            return EVO_ERR_INVALID_ARG;

    if (!aligned(LSE, 4)) return EVO_ERR_MISALIGNED;
    const int64_t int_max = 2147483647;
    // bf16 runs on the tensor-core kernel for D in {16, 32, 64, 128}; every
    // other bf16 head dim up to 128 runs on the SIMT kernel
    *tensor_core = dtype != EVO_DTYPE_FP32 && (D == 16 || D == 32 || D == 64 || D == 128);
    if (*tensor_core) {
        // TMA coordinates are 32-bit; the CTA count (query blocks x heads x
        // n pairs x batch) must fit the grid's x dimension
        int64_t ctas;
        if (bn > int_max || bh > int_max || S > int_max || N > int_max || H > int_max ||
            !mul_ok((S + evo::kBM - 1) / evo::kBM, bh, &ctas) ||
            !mul_ok(ctas, (N + evo::tri_slices(int(D)) - 1) / evo::tri_slices(int(D)), &ctas) || ctas > int_max)
            return EVO_ERR_UNSUPPORTED_SHAPE;
        // the pair bias is loaded by TMA (16-byte rule) when S % 8 == 0, else
        // element by element (2-byte rule)
        if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(O, 16) ||
            (pair_bias && !aligned(pair_bias, S % 8 == 0 ? 16 : 2)) || (mask_bias && !aligned(mask_bias, 2)))
            return EVO_ERR_MISALIGNED;
    } else {
        if (D > evo::kF32MaxD) return EVO_ERR_UNSUPPORTED_SHAPE;
        const int64_t num_qb = (S + evo::kF32Rows - 1) / evo::kF32Rows;
        int64_t blocks;
        if (!mul_ok(bnsh / S, num_qb, &blocks) || blocks > int_max || S > int_max || N > int_max || H > int_max)
            return EVO_ERR_UNSUPPORTED_SHAPE;
        if (!aligned(Q, es) || !aligned(K, es) || !aligned(V, es) || !aligned(O, es) ||
            (pair_bias && !aligned(pair_bias, es)) || (mask_bias && !aligned(mask_bias, es)))
            return EVO_ERR_MISALIGNED;
    }

    return EVO_OK;
}

// Launches the forward pass on the current device, `dev`, after check_fwd.
int launch_fwd(int dev, bool tensor_core, const void* Q, const void* K, const void* V, const void* mask_bias,
               const void* pair_bias, void* O, float* LSE, int64_t B, int64_t N, int64_t S, int64_t H, int64_t D,
               int dtype, cudaStream_t st) {
    if (dtype == EVO_DTYPE_FP32)
        return launch_f32<float>(dev, Q, K, V, mask_bias, pair_bias, O, LSE, B, N, S, H, D, st);
    if (!tensor_core)
        return dtype == EVO_DTYPE_FP16
                   ? launch_f32<__half>(dev, Q, K, V, mask_bias, pair_bias, O, LSE, B, N, S, H, D, st)
                   : launch_f32<uint16_t>(dev, Q, K, V, mask_bias, pair_bias, O, LSE, B, N, S, H, D, st);

    if (encode_fn() == nullptr) return EVO_ERR_CUDA;
    const bool has_pair = pair_bias != nullptr;
    const bool f16 = dtype == EVO_DTYPE_FP16;
#define EVO_LAUNCH_TRI(DD)                                                                                        \
    if (f16)                                                                                                      \
        return has_pair ? launch_tri<DD, true, true>(dev, Q, K, V, mask_bias, pair_bias, O, LSE, B, N, S, H, st)  \
                        : launch_tri<DD, false, true>(dev, Q, K, V, mask_bias, pair_bias, O, LSE, B, N, S, H, st); \
    return has_pair ? launch_tri<DD, true, false>(dev, Q, K, V, mask_bias, pair_bias, O, LSE, B, N, S, H, st)      \
                    : launch_tri<DD, false, false>(dev, Q, K, V, mask_bias, pair_bias, O, LSE, B, N, S, H, st)
    switch (D) {
        case 16: EVO_LAUNCH_TRI(16);
        case 32: EVO_LAUNCH_TRI(32);
        case 64: EVO_LAUNCH_TRI(64);
        default: EVO_LAUNCH_TRI(128);
    }
#undef EVO_LAUNCH_TRI
}

// Every buffer of a call must live on Q's device; makes it current.
int select_call_device(const void* Q, const void* K, const void* V, const void* O, const void* LSE,
                       const void* mask_bias, const void* pair_bias, DeviceScope& scope) {
    const int dev = select_device_of(Q, scope);
    if (dev < 0) return dev;
    if (dev >= kMaxDevices) return EVO_ERR_UNSUPPORTED_SHAPE;
    for (const void* ptr : {K, V, O, LSE, mask_bias, pair_bias})
        if (ptr != nullptr && device_of(ptr) != dev) return EVO_ERR_INVALID_ARG;
    return dev;
}

// Copy streams and events of evo_attn_fwd_host: created once per device on
// first use, kept for the life of the process, and used under `mu` so that
// concurrent calls enqueue one after the other.
struct HostPipe {
    static constexpr int kRing = 4;  // events reused round-robin across chunks
    std::mutex mu;
    bool ready = false;
    cudaStream_t h2d = nullptr, d2h = nullptr;
    cudaEvent_t start = nullptr, done = nullptr;
    cudaEvent_t in[kRing] = {}, out[kRing] = {};
};
HostPipe g_pipes[kMaxDevices];

int init_pipe(HostPipe& hp) {
    if (hp.ready) return EVO_OK;
    const unsigned ef = cudaEventDisableTiming;
    if (cudaStreamCreateWithFlags(&hp.h2d, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&hp.d2h, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&hp.start, ef) != cudaSuccess || cudaEventCreateWithFlags(&hp.done, ef) != cudaSuccess)
        return EVO_ERR_CUDA;
    for (int r = 0; r < HostPipe::kRing; ++r)
        if (cudaEventCreateWithFlags(&hp.in[r], ef) != cudaSuccess ||
            cudaEventCreateWithFlags(&hp.out[r], ef) != cudaSuccess)
            return EVO_ERR_CUDA;
    hp.ready = true;
    return EVO_OK;
}

bool page_locked(const void* p) {
    if (p == nullptr) return true;
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return attr.type == cudaMemoryTypeHost;
}

const char* at(const void* p, int64_t bytes) { return static_cast<const char*>(p) + bytes; }
char* at(void* p, int64_t bytes) { return static_cast<char*>(p) + bytes; }

}  // namespace

extern "C" EVO_API int evo_attn_fwd(const void* Q, const void* K, const void* V, const void* mask_bias,
                            const void* pair_bias, void* O, float* LSE, int64_t B, int64_t N, int64_t S, int64_t H,
                            int64_t D, int dtype, evo_stream_t stream) {
    bool tensor_core = false;
    const int st = check_fwd(Q, K, V, mask_bias, pair_bias, O, LSE, B, N, S, H, D, dtype, &tensor_core);
    if (st != EVO_OK || B == 0 || N == 0 || S == 0 || H == 0) return st;
    RelaxedCapture relaxed;
    DeviceScope scope;
    const int dev = select_call_device(Q, K, V, O, LSE, mask_bias, pair_bias, scope);
    if (dev < 0) return dev;
    return launch_fwd(dev, tensor_core, Q, K, V, mask_bias, pair_bias, O, LSE, B, N, S, H, D, dtype,
                      reinterpret_cast<cudaStream_t>(stream));
}

extern "C" EVO_API int evo_attn_sync_status(evo_stream_t stream) {
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // The status word read is the one on the stream's device (for the legacy
    // default stream: the current device), whichever device is current.
    int dev = -1;
    if (cudaStreamGetDevice(st, &dev) != cudaSuccess) return EVO_ERR_CUDA;
    DeviceScope scope;
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess) return EVO_ERR_CUDA;
    if (cur != dev) {
        if (cudaSetDevice(dev) != cudaSuccess) return EVO_ERR_CUDA;
        scope.prev = cur;
        scope.changed = true;
    }
    if (cudaStreamSynchronize(st) != cudaSuccess) return EVO_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbolAsync(&v, evo::g_status, sizeof(int), 0, cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return EVO_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return EVO_ERR_CUDA;
    if (v != 0) {
        const int zero = 0;
        if (cudaMemcpyToSymbolAsync(evo::g_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st) !=
                cudaSuccess ||
            cudaStreamSynchronize(st) != cudaSuccess)
            return EVO_ERR_CUDA;
    }
    return v;
}

extern "C" EVO_API const char* evo_attn_strerror(int status) {
    switch (status) {
        case EVO_OK: return "ok";
        case EVO_ERR_INVALID_ARG: return "invalid argument (NULL pointer, negative size or overlapping outputs)";
        case EVO_ERR_UNSUPPORTED_DTYPE: return "unsupported dtype";
        case EVO_ERR_UNSUPPORTED_SHAPE: return "shape outside the supported envelope";
        case EVO_ERR_MISALIGNED: return "a pointer breaks the alignment rule";
        case EVO_ERR_CUDA: return "a CUDA call failed";
        case EVO_ERR_TIMEOUT: return "a device-side wait timed out";
        case EVO_ERR_RANGE: return "an input value is outside the supported range (|V| > 65504 with bf16, or a non-finite output)";
        case EVO_ERR_SCRATCH: return "the problem needs more scratch than the static backward scratch holds (64 MiB)";
        default: return "unknown status";
    }
}

extern "C" EVO_API int evo_attn_version(void) { return 100; }

extern "C" EVO_API int evo_attn_fwd_host(const void* Qh, const void* Kh, const void* Vh, const void* mask_h,
                                 const void* pair_h, void* Oh, float* LSEh, void* Qd, void* Kd, void* Vd,
                                 void* mask_d, void* pair_d, void* Od, float* LSEd, int64_t B, int64_t N,
                                 int64_t S, int64_t H, int64_t D, int dtype, int64_t chunk_n,
                                 evo_stream_t stream) {
    // the device buffers get every check of evo_attn_fwd
    bool tensor_core = false;
    int st = check_fwd(Qd, Kd, Vd, mask_d, pair_d, Od, LSEd, B, N, S, H, D, dtype, &tensor_core);
    if (st != EVO_OK) return st;
    if (chunk_n < 0) return EVO_ERR_INVALID_ARG;
    if ((mask_h == nullptr) != (mask_d == nullptr) || (pair_h == nullptr) != (pair_d == nullptr))
        return EVO_ERR_INVALID_ARG;
    if (B == 0 || N == 0 || S == 0 || H == 0) return EVO_OK;
    if (!Qh || !Kh || !Vh || !Oh || !LSEh) return EVO_ERR_INVALID_ARG;
    RelaxedCapture relaxed;
    const int64_t es = dtype == EVO_DTYPE_FP32 ? 4 : 2;
    // sizes fit int64: check_fwd multiplied them out already
    const int64_t row = S * H * D * es;  // bytes of one (b, n) slice of Q, K, V or O
    const int64_t mrow = S * es, lrow = H * S * 4, prow = H * S * S * es;
    const int64_t qkv_bytes = B * N * row, lse_bytes = B * N * lrow;
    // host outputs must not overlap each other or any host input
    const void* ins[5] = {Qh, Kh, Vh, mask_h, pair_h};
    const int64_t in_bytes[5] = {qkv_bytes, qkv_bytes, qkv_bytes, B * N * mrow, B * prow};
    if (overlap(Oh, qkv_bytes, LSEh, lse_bytes)) return EVO_ERR_INVALID_ARG;
    for (int i = 0; i < 5; ++i)
        if (overlap(Oh, qkv_bytes, ins[i], in_bytes[i]) || overlap(LSEh, lse_bytes, ins[i], in_bytes[i]))
            return EVO_ERR_INVALID_ARG;
    for (const void* p : {Qh, Kh, Vh, mask_h, pair_h, static_cast<const void*>(Oh), static_cast<const void*>(LSEh)})
        if (!page_locked(p)) return EVO_ERR_INVALID_ARG;

    DeviceScope scope;
    const int dev = select_call_device(Qd, Kd, Vd, Od, LSEd, mask_d, pair_d, scope);
    if (dev < 0) return dev;
    HostPipe& hp = g_pipes[dev];
    std::lock_guard<std::mutex> lock(hp.mu);
    if (init_pipe(hp) != EVO_OK) return EVO_ERR_CUDA;

    // chunks of an even number of n slices (the tensor-core kernel pairs
    // them), about eight per batch entry by default
    int64_t cn = chunk_n > 0 ? chunk_n : 2 * ((N + 15) / 16);
    if (cn > N) cn = N;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    const cudaMemcpyKind h2d = cudaMemcpyHostToDevice, d2h = cudaMemcpyDeviceToHost;
    // the copies start after the work already on the caller's stream
    if (cudaEventRecord(hp.start, cs) != cudaSuccess || cudaStreamWaitEvent(hp.h2d, hp.start, 0) != cudaSuccess ||
        cudaStreamWaitEvent(hp.d2h, hp.start, 0) != cudaSuccess)
        return EVO_ERR_CUDA;
    int64_t i = 0;
    for (int64_t b = 0; b < B && st == EVO_OK; ++b) {
        if (pair_h && cudaMemcpyAsync(at(pair_d, b * prow), at(pair_h, b * prow), prow, h2d, hp.h2d) != cudaSuccess) {
            st = EVO_ERR_CUDA;
            break;
        }
        for (int64_t n0 = 0; n0 < N; n0 += cn, ++i) {
            const int64_t nn = (N - n0) < cn ? (N - n0) : cn;
            const int64_t bn0 = b * N + n0;
            const int r = int(i % HostPipe::kRing);
            bool ok = cudaMemcpyAsync(at(Qd, bn0 * row), at(Qh, bn0 * row), nn * row, h2d, hp.h2d) == cudaSuccess &&
                      cudaMemcpyAsync(at(Kd, bn0 * row), at(Kh, bn0 * row), nn * row, h2d, hp.h2d) == cudaSuccess &&
                      cudaMemcpyAsync(at(Vd, bn0 * row), at(Vh, bn0 * row), nn * row, h2d, hp.h2d) == cudaSuccess &&
                      (!mask_h ||
                       cudaMemcpyAsync(at(mask_d, bn0 * mrow), at(mask_h, bn0 * mrow), nn * mrow, h2d, hp.h2d) ==
                           cudaSuccess) &&
                      cudaEventRecord(hp.in[r], hp.h2d) == cudaSuccess &&
                      cudaStreamWaitEvent(cs, hp.in[r], 0) == cudaSuccess;
            if (!ok) {
                st = EVO_ERR_CUDA;
                break;
            }
            st = launch_fwd(dev, tensor_core, at(Qd, bn0 * row), at(Kd, bn0 * row), at(Vd, bn0 * row),
                            mask_d ? at(mask_d, bn0 * mrow) : nullptr, pair_d ? at(pair_d, b * prow) : nullptr,
                            at(Od, bn0 * row), reinterpret_cast<float*>(at(LSEd, bn0 * lrow)), 1, nn, S, H, D,
                            dtype, cs);
            if (st != EVO_OK) break;
            ok = cudaEventRecord(hp.out[r], cs) == cudaSuccess && cudaStreamWaitEvent(hp.d2h, hp.out[r], 0) == cudaSuccess &&
                 cudaMemcpyAsync(at(Oh, bn0 * row), at(Od, bn0 * row), nn * row, d2h, hp.d2h) == cudaSuccess &&
                 cudaMemcpyAsync(at(LSEh, bn0 * lrow), at(LSEd, bn0 * lrow), nn * lrow, d2h, hp.d2h) == cudaSuccess;
            if (!ok) {
                st = EVO_ERR_CUDA;
                break;
            }
        }
    }
    // the call ends on the caller's stream after the last copy back, on
    // error paths too, so that nothing of it is left running unordered
    if (cudaEventRecord(hp.done, hp.d2h) != cudaSuccess || cudaEventRecord(hp.in[0], hp.h2d) != cudaSuccess ||
        cudaStreamWaitEvent(cs, hp.done, 0) != cudaSuccess || cudaStreamWaitEvent(cs, hp.in[0], 0) != cudaSuccess)
        return EVO_ERR_CUDA;
    return st;
}

// ---------------------------------------------------------------- backward

namespace {

// Workspace of evo_attn_bwd: fp32 sections, each starting on a 256-byte
// boundary, in this order (byte offsets from the workspace pointer).
struct BwdLayout {
    int64_t cmask = 0;      // [B * N]        mask rebase c of each (b, n)
    int64_t lse_r = 0;      // [B, N, H, S]   LSE - c (natural log)
    int64_t delta = 0;      // [B, N, H, S]   dO . O
    int64_t dq_acc = 0;     // [B, N, S, H, D] dQ partial sums (tensor-core path)
    int64_t dmask_acc = 0;  // [B, N, S]      dmask partial sums (tensor-core path)
    int64_t dpair_acc = 0;  // [B, H, S, S]   dpair partial sums (tensor-core path)
    int64_t shifted = 0;    // [1 + B * N] int32: count and list of the (b, n) whose LSE is recomputed
    int64_t total = 0;
};

bool bwd_layout(int64_t B, int64_t N, int64_t S, int64_t H, int64_t D, BwdLayout* L) {
    int64_t bn, bns, bnhs, bnshd, bh, bhs, bhss;
    if (!mul_ok(B, N, &bn) || !mul_ok(bn, S, &bns) || !mul_ok(bns, H, &bnhs) || !mul_ok(bnhs, D, &bnshd) ||
        !mul_ok(B, H, &bh) || !mul_ok(bh, S, &bhs) || !mul_ok(bhs, S, &bhss))
        return false;
    int64_t off = 0;
    auto take = [&off](int64_t elems, int64_t* at) {
        int64_t bytes;
        if (!mul_ok(elems, 4, &bytes) || bytes > INT64_MAX - off - 256) return false;
        *at = off;
        off += (bytes + 255) / 256 * 256;
        return true;
    };
    if (!take(bn, &L->cmask) || !take(bnhs, &L->lse_r) || !take(bnhs, &L->delta) || !take(bnshd, &L->dq_acc) ||
        !take(bns, &L->dmask_acc) || !take(bhss, &L->dpair_acc) || !take(bn + 1, &L->shifted))
        return false;
    L->total = off;
    return true;
}

// Every argument check of evo_attn_bwd that needs no CUDA call, in the order
// the header lists them.  On success *tensor_core says which path runs.
int check_bwd(const void* Q, const void* K, const void* V, const void* mask_bias, const void* pair_bias,
              const void* O, const float* LSE, const void* dO, void* dQ, void* dK, void* dV, void* dmask,
              void* dpair, void* workspace, int64_t workspace_bytes, int64_t B, int64_t N, int64_t S, int64_t H,
              int64_t D, int dtype, bool* tensor_core) {
    *tensor_core = false;
    if (B < 0 || N < 0 || S < 0 || H < 0 || D < 0 || workspace_bytes < 0) return EVO_ERR_INVALID_ARG;
    if (dtype != EVO_DTYPE_BF16 && dtype != EVO_DTYPE_FP32 && dtype != EVO_DTYPE_FP16) return EVO_ERR_UNSUPPORTED_DTYPE;
    if (D == 0 || D > evo::kF32MaxD) return EVO_ERR_UNSUPPORTED_SHAPE;
    if (B == 0 || N == 0 || S == 0 || H == 0) return EVO_OK;  // nothing to compute
    if (!Q || !K || !V || !O || !LSE || !dO || !dQ || !dK || !dV || !workspace) return EVO_ERR_INVALID_ARG;
    if ((dmask && !mask_bias) || (dpair && !pair_bias)) return EVO_ERR_INVALID_ARG;

    const int64_t es = dtype == EVO_DTYPE_FP32 ? 4 : 2;
    int64_t bn, bns, bnsh, qkv_elems, qkv_bytes, mask_bytes, bh, pair_elems, pair_bytes, lse_bytes;
    if (!mul_ok(B, N, &bn) || !mul_ok(bn, S, &bns) || !mul_ok(bns, H, &bnsh) || !mul_ok(bnsh, D, &qkv_elems) ||
        !mul_ok(qkv_elems, es, &qkv_bytes) || !mul_ok(bns, es, &mask_bytes) || !mul_ok(B, H, &bh) ||
        !mul_ok(bh, S, &pair_elems) || !mul_ok(pair_elems, S, &pair_elems) ||
        !mul_ok(pair_elems, es, &pair_bytes) || !mul_ok(bnsh, 4, &lse_bytes))
        return EVO_ERR_UNSUPPORTED_SHAPE;
    BwdLayout L;
    if (!bwd_layout(B, N, S, H, D, &L)) return EVO_ERR_UNSUPPORTED_SHAPE;
    if (workspace_bytes < L.total) return EVO_ERR_INVALID_ARG;
    if (!aligned(workspace, 256)) return EVO_ERR_MISALIGNED;

    // outputs (and the workspace) must not overlap each other or any input
    const void* ins[8] = {Q, K, V, mask_bias, pair_bias, O, LSE, dO};
    const int64_t in_bytes[8] = {qkv_bytes, qkv_bytes, qkv_bytes, mask_bytes, pair_bytes, qkv_bytes, lse_bytes,
                                 qkv_bytes};
    const void* outs[6] = {dQ, dK, dV, dmask, dpair, workspace};
    const int64_t out_bytes[6] = {qkv_bytes, qkv_bytes, qkv_bytes, mask_bytes, pair_bytes, L.total};
    for (int a = 0; a < 6; ++a) {
        for (int b = a + 1; b < 6; ++b)
            if (overlap(outs[a], out_bytes[a], outs[b], out_bytes[b])) return EVO_ERR_INVALID_ARG;
        for (int i = 0; i < 8; ++i)
            if (overlap(outs[a], out_bytes[a], ins[i], in_bytes[i])) return EVO_ERR_INVALID_ARG;
    }

    if (!aligned(LSE, 4)) return EVO_ERR_MISALIGNED;
    const int64_t int_max = 2147483647;
    if (S > int_max || N > int_max || H > int_max || bn > int_max) return EVO_ERR_UNSUPPORTED_SHAPE;
    // the SIMT kernels run one thread per (slice, row, 32 columns), per
    // (b, n, key) and per pair-bias element, in blocks of 128
    const int64_t nch = (D + evo::kBwdChunk - 1) / evo::kBwdChunk;
    int64_t threads;
    if (!mul_ok(bnsh, nch, &threads) || threads / 128 >= int_max || pair_elems / 128 >= int_max)
        return EVO_ERR_UNSUPPORTED_SHAPE;
    for (const void* ptr : {Q, K, V, O, dO, static_cast<const void*>(dQ), static_cast<const void*>(dK),
                            static_cast<const void*>(dV), mask_bias, pair_bias, static_cast<const void*>(dmask),
                            static_cast<const void*>(dpair)})
        if (ptr && !aligned(ptr, uintptr_t(es))) return EVO_ERR_MISALIGNED;
    // the tensor-core path: 16-bit types, D in {16, 32, 64}, pair-bias rows in
    // whole 16-byte units (loaded by TMA), the tiles 16-byte aligned; every
    // other accepted call runs on the SIMT kernels
    int64_t units;
    *tensor_core = dtype != EVO_DTYPE_FP32 && (D == 16 || D == 32 || D == 64) &&
                   (pair_bias == nullptr || (S % 8 == 0 && aligned(pair_bias, 16))) && aligned(Q, 16) &&
                   aligned(K, 16) && aligned(V, 16) && aligned(dO, 16) && aligned(dQ, 16) && aligned(dK, 16) &&
                   aligned(dV, 16) && mul_ok(bnsh / S, (S + evo::kBN - 1) / evo::kBN, &units) && units <= int_max;
    return EVO_OK;
}

template <typename T>
evo::BwdParams<T> make_bwd_params(const void* Q, const void* K, const void* V, const void* mask_bias,
                                  const void* pair_bias, const void* O, const float* LSE, const void* dO, void* dQ,
                                  void* dK, void* dV, void* dmask, void* dpair, void* workspace, int64_t B,
                                  int64_t N, int64_t S, int64_t H, int64_t D) {
    BwdLayout L;
    bwd_layout(B, N, S, H, D, &L);  // checked by check_bwd
    char* ws = static_cast<char*>(workspace);
    evo::BwdParams<T> p;
    p.q = static_cast<const T*>(Q);
    p.k = static_cast<const T*>(K);
    p.v = static_cast<const T*>(V);
    p.mask = static_cast<const T*>(mask_bias);
    p.pair = static_cast<const T*>(pair_bias);
    p.o = static_cast<const T*>(O);
    p.dout = static_cast<const T*>(dO);
    p.lse = LSE;
    p.dq = static_cast<T*>(dQ);
    p.dk = static_cast<T*>(dK);
    p.dv = static_cast<T*>(dV);
    p.dmask = static_cast<T*>(dmask);
    p.dpair = static_cast<T*>(dpair);
    p.cmask = reinterpret_cast<float*>(ws + L.cmask);
    p.lse_r = reinterpret_cast<float*>(ws + L.lse_r);
    p.delta = reinterpret_cast<float*>(ws + L.delta);
    p.shifted = reinterpret_cast<int*>(ws + L.shifted);
    p.B = int(B);
    p.N = int(N);
    p.S = int(S);
    p.H = int(H);
    p.D = int(D);
    p.scale = float(1.0 / std::sqrt(double(D)));
    p.vec16 = (sizeof(T) == 2 && D % 8 == 0 && aligned(O, 16) && aligned(dO, 16) && aligned(K, 16)) ? 1 : 0;
    return p;
}

// The mask shift of every (b, n), then delta and the rebased LSE of every
// row (recomputed for the rows of a heavily shifted n): both paths.
template <typename T>
int launch_rowstats(int dev, const evo::BwdParams<T>& p, int64_t B, int64_t N, int64_t S, int64_t H,
                    cudaStream_t st) {
    cudaLaunchConfig_t cfg = {};
    cfg.stream = st;
    cfg.blockDim = dim3(256, 1, 1);
    const long long bns = (long long)B * N;
    if (cudaMemsetAsync(p.shifted, 0, sizeof(int), st) != cudaSuccess) return EVO_ERR_CUDA;
    cfg.gridDim = dim3(unsigned((bns + 7) / 8), 1, 1);
    if (cudaLaunchKernelEx(&cfg, evo::evo_bwd_shift_kernel<T>, p, bns) != cudaSuccess) return EVO_ERR_CUDA;
    const long long rows = bns * S * H;
    cfg.gridDim = dim3(unsigned((rows + 255) / 256), 1, 1);
    if (cudaLaunchKernelEx(&cfg, evo::evo_bwd_rowstats_kernel<T>, p, rows) != cudaSuccess) return EVO_ERR_CUDA;
    if (p.mask == nullptr) return EVO_OK;  // no shift, nothing to recompute
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
        return EVO_ERR_CUDA;
    cfg.gridDim = dim3(unsigned(4 * sms), 1, 1);
    return cudaLaunchKernelEx(&cfg, evo::evo_bwd_lse_recompute_kernel<T>, p) == cudaSuccess ? EVO_OK : EVO_ERR_CUDA;
}

template <typename T>
int launch_bwd_simt(int dev, const void* Q, const void* K, const void* V, const void* mask_bias, const void* pair_bias,
                    const void* O, const float* LSE, const void* dO, void* dQ, void* dK, void* dV, void* dmask,
                    void* dpair, void* workspace, int64_t B, int64_t N, int64_t S, int64_t H, int64_t D,
                    cudaStream_t st) {
    const evo::BwdParams<T> p = make_bwd_params<T>(Q, K, V, mask_bias, pair_bias, O, LSE, dO, dQ, dK, dV, dmask,
                                                   dpair, workspace, B, N, S, H, D);
    if (launch_rowstats<T>(dev, p, B, N, S, H, st) != EVO_OK) return EVO_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.stream = st;
    const long long nch = (D + evo::kBwdChunk - 1) / evo::kBwdChunk;
    const long long rows = (long long)B * N * H * S * nch;
    cfg.blockDim = dim3(128, 1, 1);
    cfg.gridDim = dim3(unsigned((rows + 127) / 128), 1, 1);
    if (cudaLaunchKernelEx(&cfg, evo::evo_bwd_simt_kv_kernel<T>, p, rows) != cudaSuccess) return EVO_ERR_CUDA;
    if (cudaLaunchKernelEx(&cfg, evo::evo_bwd_simt_q_kernel<T>, p, rows) != cudaSuccess) return EVO_ERR_CUDA;
    if (dmask) {
        const long long n = (long long)B * N * S;
        cfg.gridDim = dim3(unsigned((n + 127) / 128), 1, 1);
        if (cudaLaunchKernelEx(&cfg, evo::evo_bwd_simt_dmask_kernel<T>, p, n) != cudaSuccess) return EVO_ERR_CUDA;
    }
    if (dpair) {
        const long long n = (long long)B * H * S * S;
        cfg.gridDim = dim3(unsigned((n + 127) / 128), 1, 1);
        if (cudaLaunchKernelEx(&cfg, evo::evo_bwd_simt_dpair_kernel<T>, p, n) != cudaSuccess) return EVO_ERR_CUDA;
    }
    return EVO_OK;
}

// The tcgen05 backward: fp32 accumulators zeroed, row statistics, the
// persistent gradient kernel, then the rounding of the fp32 sums.
template <int D, bool HAS_PAIR, bool F16>
int launch_bwd_tri(int dev, const void* Q, const void* K, const void* V, const void* mask_bias,
                   const void* pair_bias, const void* O, const float* LSE, const void* dO, void* dQ, void* dK,
                   void* dV, void* dmask, void* dpair, void* workspace, int64_t B, int64_t N, int64_t S, int64_t H,
                   cudaStream_t st) {
    using C = evo::BwdCfg<D, HAS_PAIR, F16>;
    using T = typename std::conditional<F16, __half, uint16_t>::type;
    auto kernel = evo::evo_bwd_tri_kernel<D, HAS_PAIR, F16>;
    static AttrOnce attr;
    if (!attr.ensure(dev, kernel, C::SMEM_BYTES)) return EVO_ERR_CUDA;
    if (C::GROUPS == 2) {
        // the register hand-over (setmaxnreg) needs the whole split at launch
        cudaFuncAttributes fa;
        if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess ||
            fa.numRegs * C::THREADS < 128 * C::LOW_REGS + 3 * 128 * C::HIGH_REGS)
            return EVO_ERR_CUDA;
    }
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
        return EVO_ERR_CUDA;
    const CUtensorMapDataType dt = F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    CUtensorMap tq, tk, tv, tdo, tp, tdp, tdq;
    std::memset(&tp, 0, sizeof(tp));
    std::memset(&tdp, 0, sizeof(tdp));
    if (!encode_qkv(&tq, Q, B * N, S, H, D, 16, dt) || !encode_qkv(&tk, K, B * N, S, H, D, 16, dt) ||
        !encode_qkv(&tv, V, B * N, S, H, D, 16, dt) || !encode_qkv(&tdo, dO, B * N, S, H, D, 16, dt))
        return EVO_ERR_CUDA;
    if (HAS_PAIR && !encode_pair(&tp, pair_bias, B * H, S, dt)) return EVO_ERR_CUDA;

    BwdLayout L;
    bwd_layout(B, N, S, H, D, &L);
    char* ws = static_cast<char*>(workspace);
    const long long n_q = (long long)B * N * S * H * D, n_m = (long long)B * N * S, n_p = (long long)B * H * S * S;
    if (cudaMemsetAsync(ws + L.dq_acc, 0, size_t(n_q) * 4, st) != cudaSuccess ||
        (dmask && cudaMemsetAsync(ws + L.dmask_acc, 0, size_t(n_m) * 4, st) != cudaSuccess) ||
        (dpair && cudaMemsetAsync(ws + L.dpair_acc, 0, size_t(n_p) * 4, st) != cudaSuccess))
        return EVO_ERR_CUDA;
    const evo::BwdParams<T> bp = make_bwd_params<T>(Q, K, V, mask_bias, pair_bias, O, LSE, dO, dQ, dK, dV, dmask,
                                                    dpair, workspace, B, N, S, H, D);
    if (launch_rowstats<T>(dev, bp, B, N, S, H, st) != EVO_OK) return EVO_ERR_CUDA;

    if (HAS_PAIR && dpair) {
        // the fp32 dpair sums as a 3-D tensor {S (key), S (query), B*H}; a box
        // is 32 keys x 32 queries (128 B rows, 128 B swizzle), the tile one
        // softmax warp reduces into it per 32-key chunk
        const cuuint64_t dims[3] = {cuuint64_t(S), cuuint64_t(S), cuuint64_t(B * H)};
        const cuuint64_t strides[2] = {cuuint64_t(S * 4), cuuint64_t(S * S * 4)};
        const cuuint32_t box[3] = {32, 32, 1};
        const cuuint32_t estr[3] = {1, 1, 1};
        if (encode_fn()(&tdp, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, ws + L.dpair_acc, dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return EVO_ERR_CUDA;
    }
    {
        // the fp32 dQ sums as a 4-D tensor {D, H, S, B*N} like Q; a box is 16
        // columns of 32 rows (64 B rows, 64 B swizzle)
        const cuuint64_t dims[4] = {cuuint64_t(D), cuuint64_t(H), cuuint64_t(S), cuuint64_t(B * N)};
        const cuuint64_t strides[3] = {cuuint64_t(D * 4), cuuint64_t(H * D * 4), cuuint64_t(S * H * D * 4)};
        const cuuint32_t box[4] = {16, 1, 32, 1};
        const cuuint32_t estr[4] = {1, 1, 1, 1};
        if (encode_fn()(&tdq, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, ws + L.dq_acc, dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return EVO_ERR_CUDA;
    }
    evo::BwdTriParams p;
    p.mask = static_cast<const uint16_t*>(mask_bias);
    p.cmask = bp.cmask;
    p.lse_r = bp.lse_r;
    p.delta = bp.delta;
    p.dk = static_cast<uint16_t*>(dK);
    p.dv = static_cast<uint16_t*>(dV);
    p.dq_acc = reinterpret_cast<float*>(ws + L.dq_acc);
    p.dmask_acc = dmask ? reinterpret_cast<float*>(ws + L.dmask_acc) : nullptr;
    p.dpair_acc = dpair ? reinterpret_cast<float*>(ws + L.dpair_acc) : nullptr;
    p.N = int(N);
    p.S = int(S);
    p.H = int(H);
    p.num_kb = int((S + evo::kBN - 1) / evo::kBN);
    p.num_qb = int((S + evo::kBM - 1) / evo::kBM);
    p.num_units = int(B * N * H * p.num_kb);
    p.scale = float(1.0 / std::sqrt(double(D)));
    p.scale_log2 = float(1.4426950408889634 / std::sqrt(double(D)));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(p.num_units < sms ? p.num_units : sms), 1, 1);
    cfg.blockDim = dim3(C::THREADS, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = st;
    if (cudaLaunchKernelEx(&cfg, kernel, tq, tk, tv, tdo, tp, tdp, tdq, p) != cudaSuccess) return EVO_ERR_CUDA;

    cudaLaunchConfig_t pc = {};
    const long long work = std::max(n_q / 4, std::max(dmask ? n_m : 0ll, dpair ? n_p : 0ll));
    pc.gridDim = dim3(unsigned(std::min<long long>((work + 255) / 256, (long long)sms * 16)), 1, 1);
    pc.blockDim = dim3(256, 1, 1);
    pc.stream = st;
    return cudaLaunchKernelEx(&pc, evo::evo_bwd_post_kernel<F16>, (const float*)p.dq_acc, static_cast<uint16_t*>(dQ),
                              n_q, p.scale, (const float*)p.dmask_acc, static_cast<uint16_t*>(dmask), n_m,
                              (const float*)p.dpair_acc, static_cast<uint16_t*>(dpair), n_p) == cudaSuccess
               ? EVO_OK
               : EVO_ERR_CUDA;
}

int launch_bwd(int dev, bool tensor_core, const void* Q, const void* K, const void* V, const void* mask_bias,
               const void* pair_bias, const void* O, const float* LSE, const void* dO, void* dQ, void* dK, void* dV,
               void* dmask, void* dpair, void* workspace, int64_t B, int64_t N, int64_t S, int64_t H, int64_t D,
               int dtype, cudaStream_t st) {
    if (tensor_core) {
        if (encode_fn() == nullptr) return EVO_ERR_CUDA;
        const bool has_pair = pair_bias != nullptr, f16 = dtype == EVO_DTYPE_FP16;
#define EVO_BWD_TRI(DD, PAIR, F)                                                                              \
    return launch_bwd_tri<DD, PAIR, F>(dev, Q, K, V, mask_bias, pair_bias, O, LSE, dO, dQ, dK, dV, dmask, dpair, \
                                       workspace, B, N, S, H, st)
#define EVO_BWD_TRI_D(DD)                                 \
    if (f16) {                                            \
        if (has_pair) EVO_BWD_TRI(DD, true, true);        \
        EVO_BWD_TRI(DD, false, true);                     \
    }                                                     \
    if (has_pair) EVO_BWD_TRI(DD, true, false);           \
    EVO_BWD_TRI(DD, false, false)
        switch (D) {
            case 16: EVO_BWD_TRI_D(16);
            case 32: EVO_BWD_TRI_D(32);
            default: EVO_BWD_TRI_D(64);
        }
#undef EVO_BWD_TRI_D
#undef EVO_BWD_TRI
    }
#define EVO_BWD_SIMT(T)                                                                                         \
    return launch_bwd_simt<T>(dev, Q, K, V, mask_bias, pair_bias, O, LSE, dO, dQ, dK, dV, dmask, dpair, workspace, B, \
                              N, S, H, D, st)
    if (dtype == EVO_DTYPE_FP32) EVO_BWD_SIMT(float);
    if (dtype == EVO_DTYPE_FP16) EVO_BWD_SIMT(__half);
    EVO_BWD_SIMT(uint16_t);
#undef EVO_BWD_SIMT
}

}  // namespace

extern "C" EVO_API int64_t evo_attn_bwd_workspace_size(int64_t B, int64_t N, int64_t S, int64_t H, int64_t D) {
    if (B < 0 || N < 0 || S < 0 || H < 0 || D < 0) return EVO_ERR_INVALID_ARG;
    BwdLayout L;
    if (!bwd_layout(B, N, S, H, D, &L)) return EVO_ERR_UNSUPPORTED_SHAPE;
    return L.total;
}

extern "C" EVO_API int evo_attn_bwd(const void* Q, const void* K, const void* V, const void* mask_bias,
                                    const void* pair_bias, const void* O, const float* LSE, const void* dO,
                                    void* dQ, void* dK, void* dV, void* dmask, void* dpair, void* workspace,
                                    int64_t workspace_bytes, int64_t B, int64_t N, int64_t S, int64_t H,
                                    int64_t D, int dtype, evo_stream_t stream) {
    bool tensor_core = false;
    const int st = check_bwd(Q, K, V, mask_bias, pair_bias, O, LSE, dO, dQ, dK, dV, dmask, dpair, workspace,
                             workspace_bytes, B, N, S, H, D, dtype, &tensor_core);
    if (st != EVO_OK || B == 0 || N == 0 || S == 0 || H == 0) return st;
    RelaxedCapture relaxed;
    DeviceScope scope;
    const int dev = select_call_device(Q, K, V, O, LSE, mask_bias, pair_bias, scope);
    if (dev < 0) return dev;
    for (const void* ptr : {dO, static_cast<const void*>(dQ), static_cast<const void*>(dK),
                            static_cast<const void*>(dV), static_cast<const void*>(dmask),
                            static_cast<const void*>(dpair), static_cast<const void*>(workspace)})
        if (ptr != nullptr && device_of(ptr) != dev) return EVO_ERR_INVALID_ARG;
    return launch_bwd(dev, tensor_core, Q, K, V, mask_bias, pair_bias, O, LSE, dO, dQ, dK, dV, dmask, dpair,
                      workspace, B, N, S, H, D, dtype, reinterpret_cast<cudaStream_t>(stream));
}

// ------------------------------------------------- backward without allocation

// Scratch of evo_attn_bwd_noalloc: one static array per device, created when
// the library is loaded, so the entry point never allocates.
static __device__ __align__(256) unsigned char g_bwd_scratch[EVO_ATTN_NOALLOC_SCRATCH_BYTES];

namespace {

// The array's device address on `dev` (the current device), looked up on the
// first call for that device and kept.
int noalloc_scratch(int dev, void** out) {
    static std::mutex mu;
    static void* addr[kMaxDevices] = {};
    std::lock_guard<std::mutex> lock(mu);
    if (addr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_bwd_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return EVO_ERR_CUDA;
        }
        addr[dev] = p;
    }
    *out = addr[dev];
    return EVO_OK;
}

}  // namespace

extern "C" EVO_API int evo_attn_bwd_noalloc(const void* Q, const void* K, const void* V, const void* mask_bias,
                                            const void* pair_bias, const void* O, const float* LSE, const void* dO,
                                            void* dQ, void* dK, void* dV, void* dmask, void* dpair, int64_t B,
                                            int64_t N, int64_t S, int64_t H, int64_t D, int dtype,
                                            evo_stream_t stream) {
    if (B < 0 || N < 0 || S < 0 || H < 0 || D < 0) return EVO_ERR_INVALID_ARG;
    if (B == 0 || N == 0 || S == 0 || H == 0) {
        bool unused = false;  // the checks of an empty call, without a workspace to name
        return check_bwd(Q, K, V, mask_bias, pair_bias, O, LSE, dO, dQ, dK, dV, dmask, dpair, nullptr, 0, B, N, S,
                         H, D, dtype, &unused);
    }
    BwdLayout L;
    if (!bwd_layout(B, N, S, H, D, &L)) return EVO_ERR_UNSUPPORTED_SHAPE;
    if (L.total > EVO_ATTN_NOALLOC_SCRATCH_BYTES) return EVO_ERR_SCRATCH;
    if (!Q) return EVO_ERR_INVALID_ARG;
    RelaxedCapture relaxed;
    DeviceScope scope;
    const int dev = select_device_of(Q, scope);
    if (dev < 0) return dev;
    if (dev >= kMaxDevices) return EVO_ERR_UNSUPPORTED_SHAPE;
    void* scratch = nullptr;
    const int sst = noalloc_scratch(dev, &scratch);
    if (sst != EVO_OK) return sst;
    bool tensor_core = false;
    const int st = check_bwd(Q, K, V, mask_bias, pair_bias, O, LSE, dO, dQ, dK, dV, dmask, dpair, scratch,
                             EVO_ATTN_NOALLOC_SCRATCH_BYTES, B, N, S, H, D, dtype, &tensor_core);
    if (st != EVO_OK) return st;
    for (const void* ptr : {K, V, O, static_cast<const void*>(LSE), mask_bias, pair_bias, dO,
                            static_cast<const void*>(dQ), static_cast<const void*>(dK), static_cast<const void*>(dV),
                            static_cast<const void*>(dmask), static_cast<const void*>(dpair)})
        if (ptr != nullptr && device_of(ptr) != dev) return EVO_ERR_INVALID_ARG;
    return launch_bwd(dev, tensor_core, Q, K, V, mask_bias, pair_bias, O, LSE, dO, dQ, dK, dV, dmask, dpair, scratch,
                      B, N, S, H, D, dtype, reinterpret_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------ triangle multiplication

namespace {

// Workspace of evo_trimul: the channel-first copies of A and B and the
// channel-first result, [Bt*C, N, Np] each (Np = N rounded up to 8), on
// 256-byte boundaries.
bool trimul_layout(int64_t Bt, int64_t N, int64_t C, int64_t* section, int64_t* total) {
    const int64_t np = (N + 7) / 8 * 8;
    int64_t e, bytes;
    if (!mul_ok(Bt, C, &e) || !mul_ok(e, N, &e) || !mul_ok(e, np, &e) || !mul_ok(e, 2, &bytes) ||
        bytes > INT64_MAX / 4)
        return false;
    *section = (bytes + 255) / 256 * 256;
    *total = 3 * *section;
    return true;
}

template <bool OUTGOING, bool F16>
int launch_trimul(int dev, const void* A, const void* Bm, void* Z, void* workspace, int64_t Bt, int64_t N,
                  int64_t Cc, cudaStream_t st) {
    using Cfg = evo::TrimulCfg<OUTGOING, F16>;
    using T = typename std::conditional<F16, __half, uint16_t>::type;
    auto kernel = evo::evo_trimul_gemm_kernel<OUTGOING, F16>;
    static AttrOnce attr;
    if (!attr.ensure(dev, kernel, Cfg::SMEM_BYTES)) return EVO_ERR_CUDA;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
        return EVO_ERR_CUDA;
    int64_t section = 0, total = 0;
    trimul_layout(Bt, N, Cc, &section, &total);  // checked by the caller
    const int64_t np = (N + 7) / 8 * 8;
    char* ws = static_cast<char*>(workspace);
    T* ac = reinterpret_cast<T*>(ws);
    T* bc = reinterpret_cast<T*>(ws + section);
    T* zc = reinterpret_cast<T*>(ws + 2 * section);

    // 16-byte transposes when every row is whole 16-byte units, else 2-byte ones
    const bool vec = Cc % 8 == 0 && aligned(A, 16) && aligned(Bm, 16) && aligned(Z, 16);
    const int tw = vec ? 64 : 32;
    auto to_cfirst = vec ? evo::evo_trimul_to_cfirst_v<T> : evo::evo_trimul_to_cfirst<T>;
    auto to_clast = vec ? evo::evo_trimul_to_clast_v<T> : evo::evo_trimul_to_clast<T>;
    cudaLaunchConfig_t cfg = {};
    cfg.stream = st;
    cfg.blockDim = dim3(256, 1, 1);
    cfg.gridDim = dim3(unsigned(Bt * N), unsigned((N + tw - 1) / tw), unsigned((Cc + tw - 1) / tw));
    if (cudaLaunchKernelEx(&cfg, to_cfirst, static_cast<const T*>(A), ac, int(N), int(Cc), int(np)) != cudaSuccess ||
        cudaLaunchKernelEx(&cfg, to_cfirst, static_cast<const T*>(Bm), bc, int(N), int(Cc), int(np)) != cudaSuccess)
        return EVO_ERR_CUDA;

    // the channel matrices as a 3-D tensor {N (columns), N (rows), Bt*C}, rows
    // Np elements apart; a box is 64 x 64 (128 B rows, 128 B swizzle)
    const CUtensorMapDataType dt = F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const cuuint64_t dims[3] = {cuuint64_t(N), cuuint64_t(N), cuuint64_t(Bt * Cc)};
    const cuuint64_t strides[2] = {cuuint64_t(np * 2), cuuint64_t(N * np * 2)};
    const cuuint32_t box[3] = {64, 64, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUtensorMap ta, tb;
    if (encode_fn()(&ta, dt, 3, ac, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
        encode_fn()(&tb, dt, 3, bc, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return EVO_ERR_CUDA;
    evo::TrimulParams p;
    p.zc = reinterpret_cast<uint16_t*>(zc);
    p.N = int(N);
    p.ldz = int(np);
    p.tiles_m = int((N + 127) / 128);
    p.tiles_n = int((N + Cfg::BN - 1) / Cfg::BN);
    p.num_tiles = int(Bt * Cc * p.tiles_m * p.tiles_n);
    p.k_steps = int((N + 63) / 64);
    cudaLaunchConfig_t gc = {};
    gc.stream = st;
    gc.blockDim = dim3(Cfg::THREADS, 1, 1);
    gc.gridDim = dim3(unsigned(p.num_tiles < sms ? p.num_tiles : sms), 1, 1);
    gc.dynamicSmemBytes = Cfg::SMEM_BYTES;
    if (cudaLaunchKernelEx(&gc, kernel, ta, tb, p) != cudaSuccess) return EVO_ERR_CUDA;
    return cudaLaunchKernelEx(&cfg, to_clast, static_cast<const T*>(zc), static_cast<T*>(Z), int(N), int(Cc),
                              int(np)) == cudaSuccess
               ? EVO_OK
               : EVO_ERR_CUDA;
}

}  // namespace

extern "C" EVO_API int64_t evo_trimul_workspace_size(int64_t Bt, int64_t N, int64_t C) {
    if (Bt < 0 || N < 0 || C < 0) return EVO_ERR_INVALID_ARG;
    int64_t section, total;
    if (!trimul_layout(Bt, N, C, &section, &total)) return EVO_ERR_UNSUPPORTED_SHAPE;
    return total;
}

extern "C" EVO_API int evo_trimul(const void* A, const void* Bm, void* Z, void* workspace, int64_t workspace_bytes,
                                  int64_t Bt, int64_t N, int64_t C, int outgoing, int dtype, evo_stream_t stream) {
    if (Bt < 0 || N < 0 || C < 0 || workspace_bytes < 0 || (outgoing != 0 && outgoing != 1))
        return EVO_ERR_INVALID_ARG;
    if (dtype != EVO_DTYPE_BF16 && dtype != EVO_DTYPE_FP16)
        return EVO_ERR_UNSUPPORTED_DTYPE;
    if (Bt == 0 || N == 0 || C == 0) return EVO_OK;
    if (!A || !Bm || !Z || !workspace) return EVO_ERR_INVALID_ARG;
    int64_t section, total, elems, bytes;
    if (!trimul_layout(Bt, N, C, &section, &total) || !mul_ok(Bt, N, &elems) || !mul_ok(elems, N, &elems) ||
        !mul_ok(elems, C, &elems) || !mul_ok(elems, 2, &bytes))
        return EVO_ERR_UNSUPPORTED_SHAPE;
    if (workspace_bytes < total) return EVO_ERR_INVALID_ARG;
    const int64_t int_max = 2147483647, tiles_mn = (N + 127) / 128;
    int64_t tiles;
    if (N > int_max || C > int_max || Bt * N > int_max || (N + 31) / 32 > 65535 || (C + 31) / 32 > 65535 ||
        !mul_ok(Bt * C, tiles_mn * tiles_mn, &tiles) || tiles > int_max || Bt * C > int_max)
        return EVO_ERR_UNSUPPORTED_SHAPE;
    if (!aligned(A, 2) || !aligned(Bm, 2) || !aligned(Z, 2)) return EVO_ERR_MISALIGNED;
    if (!aligned(workspace, 256)) return EVO_ERR_MISALIGNED;
    if (overlap(Z, bytes, A, bytes) || overlap(Z, bytes, Bm, bytes) || overlap(workspace, total, A, bytes) ||
        overlap(workspace, total, Bm, bytes) || overlap(workspace, total, Z, bytes))
        return EVO_ERR_INVALID_ARG;
    RelaxedCapture relaxed;
    DeviceScope scope;
    const int dev = select_device_of(A, scope);
    if (dev < 0) return dev;
    if (dev >= kMaxDevices) return EVO_ERR_UNSUPPORTED_SHAPE;
    for (const void* ptr : {Bm, static_cast<const void*>(Z), static_cast<const void*>(workspace)})
        if (device_of(ptr) != dev) return EVO_ERR_INVALID_ARG;
    if (encode_fn() == nullptr) return EVO_ERR_CUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const bool f16 = dtype == EVO_DTYPE_FP16;
    if (outgoing)
        return f16 ? launch_trimul<true, true>(dev, A, Bm, Z, workspace, Bt, N, C, st)
                   : launch_trimul<true, false>(dev, A, Bm, Z, workspace, Bt, N, C, st);
    return f16 ? launch_trimul<false, true>(dev, A, Bm, Z, workspace, Bt, N, C, st)
               : launch_trimul<false, false>(dev, A, Bm, Z, workspace, Bt, N, C, st);
}
