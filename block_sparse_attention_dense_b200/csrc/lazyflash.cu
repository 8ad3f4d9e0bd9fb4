// Host side of the LazyFlash C ABI (include/lazyflash.h): argument checks,
// workspace sizing, TMA tensor-map encoding and kernel launches.  Nothing
// here computes attention; every step of the path runs in the kernels of
// lf_fwd.cuh, lf_select.cuh and lf_bwd.cuh.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "lazyflash.h"
#include "lf_bwd.cuh"
#include "lf_device.cuh"
#include "lf_fwd.cuh"
#include "lf_select.cuh"

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

lf_status check_desc(const lf_attn_desc* d) {
    if (!d) return LF_ERR_INVALID_ARG;
    if (d->nseq < 1 || !d->cu_seqlens || d->total_tokens < 0 || d->max_seqlen < 0)
        return LF_ERR_INVALID_ARG;
    if (d->hq < 1 || d->hkv < 1 || d->hq % d->hkv != 0) return LF_ERR_INVALID_ARG;
    if (d->hq > 65535 || d->hkv > 65535) return LF_ERR_UNSUPPORTED;
    if (!(d->softmax_scale > 0.f) || !std::isfinite(d->softmax_scale)) return LF_ERR_INVALID_ARG;
    if (d->causal != 0 && d->causal != 1) return LF_ERR_INVALID_ARG;
    if (d->d != 64 && d->d != 128) return LF_ERR_UNSUPPORTED;
    if (d->block_q != 64 && d->block_q != 128) return LF_ERR_UNSUPPORTED;
    if (d->nseq > 65535) return LF_ERR_UNSUPPORTED;
    // element offsets are computed in 64 bits; row indices in 32 bits
    if ((int64_t)d->total_tokens * d->hq > (int64_t)1 << 31) return LF_ERR_UNSUPPORTED;
    return LF_OK;
}

inline int nbmax_of(const lf_attn_desc* d) { return (d->max_seqlen + d->block_q - 1) / d->block_q; }
inline int ntiles_of(const lf_attn_desc* d) { return (d->max_seqlen + 127) / 128; }

// Backward workspace: fp32 accumulators dQ [hq][T][d] (head-major), dK and dV
// [T][hkv][d]
// (one contiguous, 256-byte aligned block, cleared by one memset), then D
// [hq][T] when the caller does not pass it.
struct BwdWs {
    size_t dq, dk, dv, acc_end, D, total;
};
inline size_t al256(size_t b) { return (b + 255) & ~size_t(255); }
BwdWs bwd_ws_layout(const lf_attn_desc* d, bool need_D) {
    BwdWs w{};
    w.dq = 0;
    w.dk = al256((size_t)d->total_tokens * d->hq * d->d * sizeof(float));
    w.dv = w.dk + al256((size_t)d->total_tokens * d->hkv * d->d * sizeof(float));
    w.acc_end = w.dv + al256((size_t)d->total_tokens * d->hkv * d->d * sizeof(float));
    w.D = w.acc_end;
    w.total = w.acc_end + (need_D ? al256((size_t)d->total_tokens * d->hq * sizeof(float)) : 0);
    return w;
}
size_t bwd_ws_bytes(const lf_attn_desc* d, bool need_D) { return bwd_ws_layout(d, need_D).total; }

// [T][H][d] bf16 -> 3-D map (d, H, T), 64 x 1 x `rows` boxes, 128-byte swizzle.
bool make_thd_map(CUtensorMap* m, const void* base, int T, int H, int D, int rows = 128) {
    EncodeTiledFn enc = encode_tiled();
    if (!enc) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T};
    const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
    const cuuint32_t box[3] = {64, 1, (cuuint32_t)rows};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [T][H][d] fp32 accumulator -> 3-D map (d, H, T), 32 x 1 x 128 boxes (128 bytes of a
// row each), 128-byte swizzle: the layout the backward stages its dK/dV tiles in.
bool make_acc_map(CUtensorMap* m, float* base, int T, int H, int D) {
    EncodeTiledFn enc = encode_tiled();
    if (!enc) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T};
    const cuuint64_t strides[2] = {(cuuint64_t)D * 4, (cuuint64_t)H * D * 4};
    const cuuint32_t box[3] = {32, 1, 128};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline lf_status launch_status() {
    return cudaGetLastError() == cudaSuccess ? LF_OK : LF_ERR_CUDA;
}

template <int D>
lf_status launch_fwd(const lf_attn_desc* d, const void* q, const void* k, const void* v, void* o,
                     float* lse, cudaStream_t st) {
    CUtensorMap mq, mk, mv;
    if (!make_thd_map(&mq, q, d->total_tokens, d->hq, D) ||
        !make_thd_map(&mk, k, d->total_tokens, d->hkv, D) ||
        !make_thd_map(&mv, v, d->total_tokens, d->hkv, D))
        return LF_ERR_CUDA;
    lf::FwdParams p{};
    p.cu_seqlens = d->cu_seqlens;
    p.T = d->total_tokens;
    p.hq = d->hq;
    p.hkv = d->hkv;
    p.causal = d->causal;
    p.max_seqlen = d->max_seqlen;
    p.nseq = d->nseq;
    p.scale_log2 = d->softmax_scale * 1.4426950408889634f;
    p.o = static_cast<__nv_bfloat16*>(o);
    p.lse = lse;
    const uint32_t smem = lf::FwdSmem<D>::kAlloc;
    if (cudaFuncSetAttribute(lf::attn_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem) != cudaSuccess)
        return LF_ERR_CUDA;
    // The kernel's warpgroups resize their register budgets (setmaxnreg); the larger
    // budget can only be granted from the registers the block was launched with, so a
    // build that launches with fewer than the budgets add up to must not run (its
    // softmax warps would wait for registers that never come).
    cudaFuncAttributes fa{};
    if (cudaFuncGetAttributes(&fa, lf::attn_fwd_kernel<D>) != cudaSuccess) return LF_ERR_CUDA;
    const int launch_regs = (fa.numRegs + 7) / 8 * 8;
    if (launch_regs * lf::kFwdThreads < 128 * lf::kFwdCtrlRegs + 256 * lf::kFwdSoftmaxRegs)
        return LF_ERR_UNSUPPORTED;
    // one CTA per pair of query tiles; the query heads of one KV head together, their
    // longest pairs first within each segment (x = pair rank * group + head in group,
    // y = KV head)
    // (x: pairs of query tiles over all segments, flattened; see segment_of_unit)
    const long long pair_units = ((long long)d->total_tokens + 255ll * d->nseq) >> 8;
    dim3 grid(static_cast<unsigned>(pair_units * (d->hq / d->hkv)), d->hkv, 1);
    // up to eight waves: every KV head's longest rows first (the whole grid's K/V then
    // shares L2, which is small at these lengths)
    int dev = 0, nsm = 148;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return LF_ERR_CUDA;
    p.tile_major = (long long)grid.x * grid.y <= 8LL * nsm ? 1 : 0;
    lf::attn_fwd_kernel<D><<<grid, lf::kFwdThreads, smem, st>>>(mq, mk, mv, p);
    return launch_status();
}

template <int D>
lf_status launch_norms(const lf_attn_desc* d, const void* dout, const void* o, float* norms,
                       float* Dv, int write_norms, cudaStream_t st) {
    dim3 grid(nbmax_of(d), d->hq, d->nseq);
    lf::norms_rowdot_kernel<D><<<grid, lf::kNormThreads, 0, st>>>(
        d->cu_seqlens, d->total_tokens, d->max_seqlen, d->hq, d->block_q, nbmax_of(d),
        static_cast<const __nv_bfloat16*>(dout), static_cast<const __nv_bfloat16*>(o), norms, Dv,
        write_norms);
    return launch_status();
}

// The backward: prologue over kept blocks (dQ accumulator rows zeroed; D computed into
// the workspace when the caller passed none), attn_bwd_kernel, dQ conversion.
template <int D>
lf_status launch_bwd(const lf_attn_desc* d, const void* q, const void* k, const void* v,
                     const void* o, const float* lse, const void* dout, const float* Dgiven,
                     const float* w, const int32_t* kidx, const int32_t* kcnt, void* dq, void* dk,
                     void* dv, void* ws, cudaStream_t st) {
    // Q and dO also in 64-row boxes: a query tile with one live half loads only that half
    CUtensorMap mq, mk, mv, mdo, mq64, mdo64;
    if (!make_thd_map(&mq, q, d->total_tokens, d->hq, D) ||
        !make_thd_map(&mk, k, d->total_tokens, d->hkv, D) ||
        !make_thd_map(&mv, v, d->total_tokens, d->hkv, D) ||
        !make_thd_map(&mdo, dout, d->total_tokens, d->hq, D) ||
        !make_thd_map(&mq64, q, d->total_tokens, d->hq, D, 64) ||
        !make_thd_map(&mdo64, dout, d->total_tokens, d->hq, D, 64))
        return LF_ERR_CUDA;
    const BwdWs lay = bwd_ws_layout(d, false);
    uint8_t* base = static_cast<uint8_t*>(ws);
    float* dq_acc = reinterpret_cast<float*>(base + lay.dq);
    float* dk_acc = reinterpret_cast<float*>(base + lay.dk);
    float* dv_acc = reinterpret_cast<float*>(base + lay.dv);
    CUtensorMap mdvacc, mdkacc;
    if (!make_acc_map(&mdvacc, dv_acc, d->total_tokens, d->hkv, D) ||
        !make_acc_map(&mdkacc, dk_acc, d->total_tokens, d->hkv, D))
        return LF_ERR_CUDA;
    // one CTA per KV tile walks the whole query group of its KV head (up to
    // kMaxHeadsPerCta heads): dK/dV are then final in TMEM and go straight to the bf16
    // outputs, with no atomics; a larger group is split over CTAs (the largest divisor
    // of the group within the limit) whose dK/dV tiles meet in fp32 accumulators
    const int group = d->hq / d->hkv;
    int heads_per_cta = group;
    while (heads_per_cta > lf::kMaxHeadsPerCta || group % heads_per_cta != 0) --heads_per_cta;
    const bool kv_direct = heads_per_cta == group;
    // the outputs (direct) or the dK/dV accumulators zeroed whole: rows no CTA writes
    // (no kept block reaches them, or outside every segment) read as 0; the dQ
    // accumulator is zeroed only in the rows of kept blocks
    const size_t nkv = (size_t)d->total_tokens * d->hkv * D;
    if (kv_direct) {
        if (cudaMemsetAsync(dk, 0, nkv * 2, st) != cudaSuccess ||
            cudaMemsetAsync(dv, 0, nkv * 2, st) != cudaSuccess)
            return LF_ERR_CUDA;
    } else if (cudaMemsetAsync(base + lay.dk, 0, lay.acc_end - lay.dk, st) != cudaSuccess) {
        return LF_ERR_CUDA;
    }
    const dim3 blocks(nbmax_of(d), d->hq, d->nseq);
    float* Dw = Dgiven ? nullptr : reinterpret_cast<float*>(base + bwd_ws_layout(d, true).D);
    lf::bwd_prologue_kernel<D><<<blocks, lf::kNormThreads, 0, st>>>(
        d->cu_seqlens, d->total_tokens, d->max_seqlen, d->hq, d->block_q, nbmax_of(d), w, dq_acc,
        static_cast<const __nv_bfloat16*>(dout), static_cast<const __nv_bfloat16*>(o), Dw);
    if (launch_status() != LF_OK) return LF_ERR_CUDA;
    const float* Dv = Dgiven ? Dgiven : Dw;
    lf::BwdParams p{};
    p.cu_seqlens = d->cu_seqlens;
    p.T = d->total_tokens;
    p.hq = d->hq;
    p.hkv = d->hkv;
    p.causal = d->causal;
    p.block_q = d->block_q;
    p.nbmax = nbmax_of(d);
    p.max_seqlen = d->max_seqlen;
    p.heads_per_cta = heads_per_cta;
    p.kv_out_direct = kv_direct ? 1 : 0;
    p.dk_out = static_cast<__nv_bfloat16*>(dk);
    p.dv_out = static_cast<__nv_bfloat16*>(dv);
    p.scale = d->softmax_scale;
    p.scale_log2 = d->softmax_scale * 1.4426950408889634f;
    p.lse = lse;
    p.Dvec = Dv;
    p.block_weight = w;
    p.kept_idx = kidx;
    p.kept_cnt = kcnt;
    p.dq_acc = dq_acc;
    const uint32_t smem = lf::BwdSmem<D>::kAlloc;
    // 64-row selection blocks: the variant that skips a tile's dropped half
    auto kern = d->block_q == 64 ? lf::attn_bwd_kernel<D, true> : lf::attn_bwd_kernel<D, false>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return LF_ERR_CUDA;
    dim3 grid(ntiles_of(d), d->hq / p.heads_per_cta, d->nseq);
    // up to eight waves of CTAs per segment (16K tokens at 8 KV heads): every head
    // group's heavy tiles first; longer segments run one group at a time, which keeps
    // the group's Q, dO and dQ accumulator in L2 (the other order was slower at 32K)
    int dev = 0, nsm = 148;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return LF_ERR_CUDA;
    p.tile_major = (long long)grid.x * grid.y <= 8LL * nsm ? 1 : 0;
    kern<<<grid, lf::kBwdThreads, smem, st>>>(mq, mk, mv, mdo, mdvacc, mdkacc, mq64, mdo64, p);
    if (launch_status() != LF_OK) return LF_ERR_CUDA;
    // fp32 accumulators -> bf16 results (dQ and dK take the softmax scale)
    const size_t nkv8 = (size_t)d->total_tokens * d->hkv * D / 8;
    const int bkv = (int)std::min<size_t>((nkv8 + 255) / 256, 148 * 16);
    lf::dq_acc_to_thd_kept_kernel<D><<<blocks, 256, 0, st>>>(d->cu_seqlens, d->total_tokens, d->max_seqlen,
                                                             d->hq, d->block_q, nbmax_of(d), w, dq_acc,
                                                             static_cast<uint4*>(dq), d->softmax_scale);
    if (!kv_direct) {
        lf::dq_convert_kernel<<<bkv, 256, 0, st>>>(reinterpret_cast<const float4*>(dk_acc),
                                                   static_cast<uint4*>(dk), nkv8, d->softmax_scale);
        lf::dq_convert_kernel<<<bkv, 256, 0, st>>>(reinterpret_cast<const float4*>(dv_acc),
                                                   static_cast<uint4*>(dv), nkv8, 1.0f);
    }
    return launch_status();
}

}  // namespace

namespace lf {
// Failure-detection self-test: one thread waits, with the kernels' bounded wait,
// on a barrier phase that nothing completes.  The wait gives up after `limit`
// cycles and records a timeout in the device flag; nothing faults or traps.
__global__ void watchdog_selftest_kernel(long long limit) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) (void)mbar_wait(&bar, 0, 99, limit);
    __syncthreads();
}
// Enqueued at the end of every call that launches kernels: copies the failure flag,
// once set, into the host-mapped page, so that the next call sees it without a
// synchronization.
__global__ void mirror_error_kernel() {
    const int e = *reinterpret_cast<volatile int*>(&g_device_error);
    int* m = g_error_mirror;
    if (e != 0 && m) {
        *reinterpret_cast<volatile int*>(m) = e;
        __threadfence_system();
    }
}
}  // namespace lf

// Scratch of lf_attn_bwd_static_ws: one array per device, loaded with the
// library and kept until the process exits.  Host code must not use this name
// as a device address (it names a host-side stand-in); the device address comes
// from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char lf_static_ws[LF_STATIC_WS_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_static_ws_mutex;
void* g_static_ws_ptr[kMaxDevices] = {};

// Device address of lf_static_ws on the current device (looked up once per device).
lf_status static_ws_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LF_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_static_ws_mutex);
    if (!g_static_ws_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, lf_static_ws) != cudaSuccess || !p) return LF_ERR_CUDA;
        g_static_ws_ptr[dev] = p;
    }
    *out = g_static_ws_ptr[dev];
    return LF_OK;
}

// Device-side errors (an expired bounded wait, a bad segment table) are recorded in
// lf::g_device_error on the device and, through lf::g_error_mirror, in this page of
// host memory, page-locked and mapped into the device address space.  Every entry
// point reads it (a plain host load, no synchronization) and reports an earlier
// call's failure before launching anything; lf_sync_status clears it.
alignas(4096) volatile int g_host_error_page[1024];
std::once_flag g_register_once;
bool g_page_mapped = false;
bool g_mirror_ready[kMaxDevices] = {};

// Once per process: map the page; once per device: tell the device where it is.
lf_status prepare_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LF_ERR_CUDA;
    std::call_once(g_register_once, [] {
        g_page_mapped = cudaHostRegister(const_cast<int*>(g_host_error_page), sizeof(g_host_error_page),
                                         cudaHostRegisterMapped | cudaHostRegisterPortable) ==
                        cudaSuccess;
        if (!g_page_mapped) (void)cudaGetLastError();
    });
    std::lock_guard<std::mutex> lock(g_static_ws_mutex);
    if (!g_mirror_ready[dev]) {
        int* dptr = nullptr;
        if (g_page_mapped) {
            void* p = nullptr;
            if (cudaHostGetDevicePointer(&p, const_cast<int*>(g_host_error_page), 0) != cudaSuccess)
                return LF_ERR_CUDA;
            dptr = static_cast<int*>(p);
        }
        if (cudaMemcpyToSymbol(lf::g_error_mirror, &dptr, sizeof(dptr)) != cudaSuccess)
            return LF_ERR_CUDA;
        g_mirror_ready[dev] = true;
    }
    return LF_OK;
}

// The call's kernels, then the flag's copy to the host page (stream order).
lf_status mirror_after(lf_status launched, cudaStream_t s) {
    if (launched != LF_OK) return launched;
    lf::mirror_error_kernel<<<1, 1, 0, s>>>();
    return launch_status();
}

lf_status status_of_device_code(int code) {
    if (code == 0) return LF_OK;
    return (code & 0xff) == lf::kErrTimeout ? LF_ERR_TIMEOUT : LF_ERR_INVALID_ARG;
}

// An earlier call's device-side failure not yet cleared by lf_sync_status.
lf_status pending_device_error() { return status_of_device_code(g_host_error_page[0]); }

}  // namespace

extern "C" {

const char* lf_status_string(lf_status s) {
    switch (s) {
        case LF_OK: return "LF_OK";
        case LF_ERR_INVALID_ARG: return "LF_ERR_INVALID_ARG: invalid argument";
        case LF_ERR_UNSUPPORTED: return "LF_ERR_UNSUPPORTED: shape not supported by this build";
        case LF_ERR_WORKSPACE: return "LF_ERR_WORKSPACE: workspace too small";
        case LF_ERR_CUDA: return "LF_ERR_CUDA: CUDA call failed";
        case LF_ERR_TIMEOUT: return "LF_ERR_TIMEOUT: a device-side bounded wait expired";
    }
    return "unknown lf_status";
}

lf_status lf_workspace_size(const lf_attn_desc* desc, int which, size_t* bytes) {
    lf_status st = check_desc(desc);
    if (st != LF_OK) return st;
    if (!bytes) return LF_ERR_INVALID_ARG;
    switch (which) {
        case LF_WS_FWD: *bytes = 0; return LF_OK;
        case LF_WS_SELECT: *bytes = 0; return LF_OK;
        case LF_WS_BWD: *bytes = bwd_ws_bytes(desc, true); return LF_OK;
    }
    return LF_ERR_INVALID_ARG;
}

lf_status lf_attn_fwd(const lf_attn_desc* desc, const void* q, const void* k, const void* v,
                      void* o, float* lse, void* ws, size_t ws_bytes, lf_stream_t stream) {
    (void)ws;
    (void)ws_bytes;
    lf_status st = check_desc(desc);
    if (st != LF_OK) return st;
    if (!q || !k || !v || !o || !lse) return LF_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return LF_ERR_INVALID_ARG;
    if ((st = pending_device_error()) != LF_OK) return st;
    if (desc->total_tokens == 0 || desc->max_seqlen == 0) return LF_OK;
    if ((st = prepare_device()) != LF_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return mirror_after(desc->d == 128 ? launch_fwd<128>(desc, q, k, v, o, lse, s)
                                       : launch_fwd<64>(desc, q, k, v, o, lse, s), s);
}

static lf_status block_select_impl(const lf_attn_desc* desc, const void* dout, const void* o,
                                   int rule, double param, uint64_t seed, uint64_t step,
                                   uint32_t flags, float* block_norm, float* D, double* tau,
                                   float* block_weight, uint8_t* keep, int32_t* kept_idx,
                                   int32_t* kept_cnt, lf_stream_t stream) {
    lf_status st = check_desc(desc);
    if (st != LF_OK) return st;
    if (rule == LF_RULE_BUDGET) {
        if (!(param >= 0.0 && param < 1.0)) return LF_ERR_INVALID_ARG;
    } else if (rule == LF_RULE_FIXED_FRACTION || rule == LF_RULE_TOPK) {
        if (!(param > 0.0 && param <= 1.0)) return LF_ERR_INVALID_ARG;
    } else {
        return LF_ERR_INVALID_ARG;
    }
    if (flags & ~LF_SELECT_NORMS_GIVEN) return LF_ERR_INVALID_ARG;
    const bool norms_given = (flags & LF_SELECT_NORMS_GIVEN) != 0;
    // dout is needed for the norms, o only for D
    if ((!norms_given && !dout) || (D && (!dout || !o)) || !block_norm || !tau || !block_weight ||
        !keep || !kept_idx || !kept_cnt)
        return LF_ERR_INVALID_ARG;
    const void* ptrs[] = {dout, o, block_norm, D, tau, block_weight, keep, kept_idx, kept_cnt};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return LF_ERR_INVALID_ARG;
    if ((st = pending_device_error()) != LF_OK) return st;
    if (desc->max_seqlen == 0) return LF_OK;
    const int nbmax = nbmax_of(desc);
    if ((size_t)nbmax * sizeof(double) > 200 * 1024) return LF_ERR_UNSUPPORTED;
    if ((st = prepare_device()) != LF_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int write_norms = norms_given ? 0 : 1;
    if (write_norms || D) {
        st = desc->d == 128 ? launch_norms<128>(desc, dout, o, block_norm, D, write_norms, s)
                            : launch_norms<64>(desc, dout, o, block_norm, D, write_norms, s);
        if (st != LF_OK) return st;
    }
    const size_t smem = (size_t)nbmax * sizeof(float);
    auto kern = rule == LF_RULE_BUDGET ? lf::select_kernel<0>
              : rule == LF_RULE_FIXED_FRACTION ? lf::select_kernel<1> : lf::select_kernel<2>;
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
        return LF_ERR_CUDA;
    dim3 grid(desc->hq, desc->nseq);
    kern<<<grid, lf::kSelectThreads, smem, s>>>(desc->cu_seqlens, desc->total_tokens, desc->max_seqlen, desc->hq,
                                desc->block_q, nbmax, block_norm, param, seed, step, tau,
                                block_weight, keep, kept_idx, kept_cnt);
    return mirror_after(launch_status(), s);
}

lf_status lf_block_select(const lf_attn_desc* desc, const void* dout, const void* o, double delta,
                          uint64_t seed, uint64_t step, uint32_t flags, float* block_norm,
                          float* D, double* tau, float* block_weight, uint8_t* keep,
                          int32_t* kept_idx, int32_t* kept_cnt, void* ws, size_t ws_bytes,
                          lf_stream_t stream) {
    (void)ws;
    (void)ws_bytes;
    return block_select_impl(desc, dout, o, LF_RULE_BUDGET, delta, seed, step, flags, block_norm,
                             D, tau, block_weight, keep, kept_idx, kept_cnt, stream);
}

lf_status lf_block_select_rule(const lf_attn_desc* desc, const void* dout, const void* o,
                               int rule, double param, uint64_t seed, uint64_t step,
                               uint32_t flags, float* block_norm, float* D, double* tau,
                               float* block_weight, uint8_t* keep, int32_t* kept_idx,
                               int32_t* kept_cnt, void* ws, size_t ws_bytes, lf_stream_t stream) {
    (void)ws;
    (void)ws_bytes;
    return block_select_impl(desc, dout, o, rule, param, seed, step, flags, block_norm, D, tau,
                             block_weight, keep, kept_idx, kept_cnt, stream);
}

lf_status lf_attn_bwd(const lf_attn_desc* desc, const void* q, const void* k, const void* v,
                      const void* o, const float* lse, const void* dout, const float* D,
                      const float* block_weight, const int32_t* kept_idx,
                      const int32_t* kept_cnt, void* dq, void* dk, void* dv, void* ws,
                      size_t ws_bytes, lf_stream_t stream) {
    lf_status st = check_desc(desc);
    if (st != LF_OK) return st;
    if (!q || !k || !v || !lse || !dout || !block_weight || !kept_idx || !kept_cnt || !dq ||
        !dk || !dv)
        return LF_ERR_INVALID_ARG;
    if (!D && !o) return LF_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, lse, dout, block_weight, kept_idx, kept_cnt, dq, dk, dv, ws};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return LF_ERR_INVALID_ARG;
    if ((o && !aligned16(o)) || (D && !aligned16(D))) return LF_ERR_INVALID_ARG;
    if ((st = pending_device_error()) != LF_OK) return st;
    if (desc->total_tokens == 0 || desc->max_seqlen == 0) return LF_OK;
    if (!ws || ws_bytes < bwd_ws_bytes(desc, D == nullptr)) return LF_ERR_WORKSPACE;
    if ((st = prepare_device()) != LF_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return mirror_after(desc->d == 128 ? launch_bwd<128>(desc, q, k, v, o, lse, dout, D, block_weight,
                                                         kept_idx, kept_cnt, dq, dk, dv, ws, s)
                                       : launch_bwd<64>(desc, q, k, v, o, lse, dout, D, block_weight,
                                                        kept_idx, kept_cnt, dq, dk, dv, ws, s),
                        s);
}

lf_status lf_attn_bwd_static_ws(const lf_attn_desc* desc, const void* q, const void* k,
                                const void* v, const void* o, const float* lse, const void* dout,
                                const float* D, const float* block_weight,
                                const int32_t* kept_idx, const int32_t* kept_cnt, void* dq,
                                void* dk, void* dv, lf_stream_t stream) {
    lf_status st = check_desc(desc);
    if (st != LF_OK) return st;
    if (!q || !k || !v || !lse || !dout || !block_weight || !kept_idx || !kept_cnt || !dq ||
        !dk || !dv)
        return LF_ERR_INVALID_ARG;
    if (!D && !o) return LF_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, lse, dout, block_weight, kept_idx, kept_cnt, dq, dk, dv};
    for (const void* p : ptrs)
        if (!aligned16(p)) return LF_ERR_INVALID_ARG;
    if ((o && !aligned16(o)) || (D && !aligned16(D))) return LF_ERR_INVALID_ARG;
    const size_t need = bwd_ws_bytes(desc, D == nullptr);
    if (need > LF_STATIC_WS_BYTES) return LF_ERR_WORKSPACE;
    if ((st = pending_device_error()) != LF_OK) return st;
    if (desc->total_tokens == 0 || desc->max_seqlen == 0) return LF_OK;
    if ((st = prepare_device()) != LF_OK) return st;
    void* ws = nullptr;
    st = static_ws_address(&ws);
    if (st != LF_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // launch_bwd clears the accumulators it uses before the kernel
    return mirror_after(desc->d == 128 ? launch_bwd<128>(desc, q, k, v, o, lse, dout, D, block_weight,
                                                         kept_idx, kept_cnt, dq, dk, dv, ws, s)
                                       : launch_bwd<64>(desc, q, k, v, o, lse, dout, D, block_weight,
                                                        kept_idx, kept_cnt, dq, dk, dv, ws, s),
                        s);
}

lf_status lf_watchdog_selftest(uint32_t limit_log2, lf_stream_t stream) {
    if (limit_log2 < 10 || limit_log2 > 31) return LF_ERR_INVALID_ARG;
    lf_status st = pending_device_error();
    if (st != LF_OK) return st;
    if ((st = prepare_device()) != LF_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    lf::watchdog_selftest_kernel<<<1, 32, 0, s>>>(1ll << limit_log2);
    return mirror_after(launch_status(), s);
}

lf_status lf_sync_status(lf_stream_t stream) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return LF_ERR_CUDA;
    int flag = 0;
    if (cudaMemcpyFromSymbol(&flag, lf::g_device_error, sizeof(int)) != cudaSuccess)
        return LF_ERR_CUDA;
    if (flag != 0) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(lf::g_device_error, &zero, sizeof(int)) != cudaSuccess)
            return LF_ERR_CUDA;
    }
    // the page may also hold a failure recorded on another device
    const int host = g_host_error_page[0];
    g_host_error_page[0] = 0;
    return status_of_device_code(flag != 0 ? flag : host);
}

lf_status lf_check_device_error(lf_stream_t stream) { return lf_sync_status(stream); }

}  // extern "C"
