// Host side of the C ABI declared in include/varlen_attn.h: argument
// validation, stream-ordered workspace, tensor maps and kernel launches.
// The whole library is this one translation unit.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <climits>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "backward_sm100.cuh"
#include "decode.cuh"
#include "prefill_sm100.cuh"
#include "schedule_build.cuh"
#include "varlen_attn.h"

namespace va {

// Failure-path probe: one thread waits, through the bounded wait every kernel
// of the library uses, on a barrier phase that nothing completes (no thread
// arrives on it).  The wait gives up after its limit, raises the timeout bit
// in the status word and the kernel returns normally.
__global__ void wait_timeout_probe_kernel(int32_t* gave_up) {
    __shared__ uint64_t bar;
    __shared__ volatile int abort_flag;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
    *gave_up = mbar_wait(&bar, 0, &abort_flag, &g_va_status) ? 0 : 1;
}

}  // namespace va

namespace {

thread_local char g_last_error[512] = "";

int fail(int code, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
    return code;
}

int cuda_fail(cudaError_t e, const char* what) {
    return fail(VA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

#define VA_CUDA(call)                                        \
    do {                                                     \
        cudaError_t e_ = (call);                             \
        if (e_ != cudaSuccess) return cuda_fail(e_, #call);  \
    } while (0)

constexpr int kMaxDevices = 64;

// Kernels this library has launched in this process (every device and thread):
// a diagnostic for counting the launches of a timed region.
std::atomic<unsigned long long> g_launches{0};
void note_launches(unsigned n) { g_launches.fetch_add(n, std::memory_order_relaxed); }
// Host-buffer entry point: up to this many pipelined chunks, once the inputs
// reach this size.
constexpr int kHostChunks = 16;
constexpr size_t kHostChunkMinBytes = size_t(8) << 20;
// ... and no chunk below this many query rows (each chunk is its own launch)
constexpr long long kHostChunkMinRows = 4096;

// Shared-memory limits of every prefill kernel variant.
int set_prefill_attributes() {
    VA_CUDA(cudaFuncSetAttribute(va::prefill_fwd_kernel<64, va::ElemBf16, false>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 va::PrefillSmem<64, va::ElemBf16>::kAlloc));
    VA_CUDA(cudaFuncSetAttribute(va::prefill_fwd_kernel<64, va::ElemBf16, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 va::PrefillSmem<64, va::ElemBf16>::kAlloc));
    VA_CUDA(cudaFuncSetAttribute(va::prefill_fwd_kernel<128, va::ElemBf16, false>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 va::PrefillSmem<128, va::ElemBf16>::kAlloc));
    VA_CUDA(cudaFuncSetAttribute(va::prefill_fwd_kernel<128, va::ElemBf16, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 va::PrefillSmem<128, va::ElemBf16>::kAlloc));
    VA_CUDA(cudaFuncSetAttribute(va::prefill_fwd_kernel<128, va::ElemE4m3, false>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 va::PrefillSmem<128, va::ElemE4m3>::kAlloc));
    return VA_OK;
}

struct DeviceInfo {
    bool ready = false;
    int num_sms = 0;
    // Library-private stream-ordered pool.  Its release threshold is
    // unlimited, so a synchronisation does not hand its memory back to the OS
    // and the next call does not pay for mapping it again.
    cudaMemPool_t pool = nullptr;
    // Copy streams of the host-buffer entry point (created on first use).
    cudaStream_t copy_in = nullptr, copy_out = nullptr;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int device_setup(int& dev, DeviceInfo*& info) {
    VA_CUDA(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) return fail(VA_ERR_UNSUPPORTED, "device ordinal %d", dev);
    std::lock_guard<std::mutex> lock(g_dev_mu);
    info = &g_dev[dev];
    if (info->ready) return VA_OK;
    cudaDeviceProp prop;
    VA_CUDA(cudaGetDeviceProperties(&prop, dev));
    if (prop.major != 10)
        return fail(VA_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a",
                    dev, prop.major, prop.minor);
    info->num_sms = prop.multiProcessorCount;
    if (!g_encode) {
        cudaDriverEntryPointQueryResult q;
        void* fn = nullptr;
        VA_CUDA(cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q));
        if (q != cudaDriverEntryPointSuccess || !fn)
            return fail(VA_ERR_CUDA, "cuTensorMapEncodeTiled entry point not found");
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    if (set_prefill_attributes() != VA_OK) return VA_ERR_CUDA;
    VA_CUDA(cudaFuncSetAttribute(va::build_schedule_kernel,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 va::kSortCapacity * 8));
    VA_CUDA(cudaFuncSetAttribute(va::build_bwd_list_kernel,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 va::kSortCapacity * 8));
    VA_CUDA(cudaFuncSetAttribute(va::bwd_dkdv_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 va::BwdSmem<64, false>::kAlloc));
    VA_CUDA(cudaFuncSetAttribute(va::bwd_dkdv_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 va::BwdSmem<128, false>::kAlloc));
    VA_CUDA(cudaFuncSetAttribute(va::bwd_dq_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 va::BwdSmem<64, true>::kAlloc));
    VA_CUDA(cudaFuncSetAttribute(va::bwd_dq_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 va::BwdSmem<128, true>::kAlloc));
    VA_CUDA(cudaFuncSetAttribute(va::decode_stream_kernel<64>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 va::DecodeSmem<64>::kAlloc));
    VA_CUDA(cudaFuncSetAttribute(va::decode_stream_kernel<128>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 va::DecodeSmem<128>::kAlloc));
    VA_CUDA(cudaFuncSetAttribute(va::decode_stream_kernel<64>,
                                 cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared));
    VA_CUDA(cudaFuncSetAttribute(va::decode_stream_kernel<128>,
                                 cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared));
    cudaMemPoolProps props = {};
    props.allocType = cudaMemAllocationTypePinned;
    props.handleTypes = cudaMemHandleTypeNone;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    VA_CUDA(cudaMemPoolCreate(&info->pool, &props));
    unsigned long long threshold = ~0ull;
    VA_CUDA(cudaMemPoolSetAttribute(info->pool, cudaMemPoolAttrReleaseThreshold, &threshold));
    info->ready = true;
    return VA_OK;
}

// Stream-ordered workspace from the library pool of the current device.
cudaError_t ws_alloc(void** p, size_t bytes, cudaStream_t stream) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices || !g_dev[dev].pool) return cudaErrorInitializationError;
    return cudaMallocFromPoolAsync(p, bytes, g_dev[dev].pool, stream);
}

// 2-D view [rows][cols] (cols contiguous) of bf16 (elem_bytes 2) or 8-bit
// (elem_bytes 1) elements; boxes of 128 bytes x box_rows, 128-byte swizzle.
int make_tile_map(CUtensorMap* map, const void* base, long long cols, long long rows, int box_rows,
                  int elem_bytes = 2) {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * elem_bytes};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / elem_bytes), static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    const CUtensorMapDataType dtype =
        elem_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    CUresult r = g_encode(map, dtype, 2, const_cast<void*>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(VA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return VA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The packed layout's preconditions on one host cu_seqlens array (boostr
// varlen_attention.rs, VarLenAttentionOps docs, "Layout contract": cumulative
// lengths starting at 0): c[0] == 0, never decreasing, no step above
// max_seqlen and, when total >= 0, c[batch] == total.  Reads entries
// 0..batch only.
int check_cu_seqlens_host(const int32_t* c, int batch, int max_seqlen, long long total,
                          const char* name) {
    if (c[0] != 0) return fail(VA_ERR_INVALID_ARG, "%s[0] = %d, must be 0", name, c[0]);
    for (int b = 0; b < batch; ++b) {
        const long long len = static_cast<long long>(c[b + 1]) - c[b];
        if (len < 0)
            return fail(VA_ERR_INVALID_ARG, "%s decreases at entry %d (%d -> %d)", name, b + 1,
                        c[b], c[b + 1]);
        if (len > max_seqlen)
            return fail(VA_ERR_INVALID_ARG, "sequence %d has length %lld > max_seqlen %d (%s)", b,
                        len, max_seqlen, name);
    }
    if (total >= 0 && c[batch] != total)
        return fail(VA_ERR_INVALID_ARG, "%s[%d] = %d, expected the total %lld", name, batch,
                    c[batch], total);
    return VA_OK;
}

struct Args {
    const void *q, *k, *v;
    const int32_t *cu_q, *cu_k;
    int batch, H, H_kv, max_q, max_k, D, causal, window;
    void* out;
    float* lse;
    const int32_t* seqused_k = nullptr;  // key counts of a capacity-strided cache, or NULL
    // E4M3 inputs and output with per-tensor scales (varlen_attention_fwd_fp8)
    int fp8 = 0;
    float q_scale = 1.f, k_scale = 1.f, v_scale = 1.f, o_scale = 1.f;
};

int validate(const Args& a) {
    if (a.batch < 0) return fail(VA_ERR_INVALID_ARG, "batch must be >= 0 (got %d)", a.batch);
    if (a.H < 1) return fail(VA_ERR_INVALID_ARG, "num_heads must be >= 1 (got %d)", a.H);
    if (a.H_kv < 1) return fail(VA_ERR_INVALID_ARG, "num_kv_heads must be >= 1 (got %d)", a.H_kv);
    if (a.H % a.H_kv != 0)
        return fail(VA_ERR_INVALID_ARG, "num_heads (%d) must be a multiple of num_kv_heads (%d)",
                    a.H, a.H_kv);
    if (a.D != 64 && a.D != 128)
        return fail(VA_ERR_UNSUPPORTED, "head_dim must be 64 or 128 (got %d)", a.D);
    if (a.window < 0) return fail(VA_ERR_INVALID_ARG, "window must be >= 0 (got %d)", a.window);
    if (a.fp8) {
        if (a.D != 128)
            return fail(VA_ERR_UNSUPPORTED, "E4M3 inputs need head_dim 128 (got %d)", a.D);
        const float sc[4] = {a.q_scale, a.k_scale, a.v_scale, a.o_scale};
        const char* nm[4] = {"q_scale", "k_scale", "v_scale", "o_scale"};
        for (int i = 0; i < 4; ++i)
            if (!(std::isfinite(sc[i]) && sc[i] > 0.f))
                return fail(VA_ERR_INVALID_ARG, "%s must be finite and > 0 (got %g)", nm[i], sc[i]);
    }
    if (a.max_q < 0 || a.max_k < 0)
        return fail(VA_ERR_INVALID_ARG, "max_seqlen_q/k must be >= 0 (got %d, %d)", a.max_q, a.max_k);
    if (a.batch == 0 || a.max_q == 0) return VA_OK;
    const char* names[] = {"q", "k", "v", "cu_seqlens_q", "cu_seqlens_k", "out", "lse"};
    const void* ptrs[] = {a.q, a.k, a.v, a.cu_q, a.cu_k, a.out, a.lse};
    for (int i = 0; i < 7; ++i)
        if (!ptrs[i]) return fail(VA_ERR_INVALID_ARG, "%s is NULL", names[i]);
    if (!aligned16(a.q) || !aligned16(a.k) || !aligned16(a.v) || !aligned16(a.out))
        return fail(VA_ERR_INVALID_ARG, "q, k, v and out must be 16-byte aligned");
    if (reinterpret_cast<uintptr_t>(a.lse) & 3u) return fail(VA_ERR_INVALID_ARG, "lse must be 4-byte aligned");
    const long long rows_q = static_cast<long long>(a.batch) * a.max_q;
    const long long rows_k = static_cast<long long>(a.batch) * a.max_k;
    if (rows_q * a.H * (long long)a.D >= (1ll << 40) || rows_k * a.H_kv * (long long)a.D >= (1ll << 40))
        return fail(VA_ERR_UNSUPPORTED, "tensors beyond 2^40 elements");
    return VA_OK;
}

// Tensor maps of the prefill kernel: Q, K, V as [rows][heads * D] with an
// upper-bound row extent (batch * max_seqlen), 128-row and 8-row boxes.
int make_prefill_maps(const Args& a, va::PrefillMaps* m) {
    const long long rows_q = std::max(1ll, static_cast<long long>(a.batch) * a.max_q);
    const long long rows_k = std::max(1ll, static_cast<long long>(a.batch) * a.max_k);
    const long long cols_q = static_cast<long long>(a.H) * a.D;
    const long long cols_k = static_cast<long long>(a.H_kv) * a.D;
    const int eb = a.fp8 ? 1 : 2;
    int rc;
    if ((rc = make_tile_map(&m->q, a.q, cols_q, rows_q, va::kBlockM, eb)) != VA_OK ||
        (rc = make_tile_map(&m->k, a.k, cols_k, rows_k, va::kBlockN, eb)) != VA_OK ||
        (rc = make_tile_map(&m->v, a.v, cols_k, rows_k, va::kBlockN, eb)) != VA_OK ||
        (rc = make_tile_map(&m->q8, a.q, cols_q, rows_q, 8, eb)) != VA_OK ||
        (rc = make_tile_map(&m->k8, a.k, cols_k, rows_k, 8, eb)) != VA_OK ||
        (rc = make_tile_map(&m->v8, a.v, cols_k, rows_k, 8, eb)) != VA_OK)
        return rc;
    return VA_OK;
}

// Kernel parameters shared by both prefill entry paths (list and workspace
// filled in by the caller).
va::PrefillParams prefill_params(const Args& a) {
    va::PrefillParams p;
    p.cu_q = a.cu_q;
    p.cu_k = a.cu_k;
    p.seqused_k = a.seqused_k;
    p.batch = a.batch;
    p.H = a.H;
    p.H_kv = a.H_kv;
    p.causal = a.causal;
    p.window = a.window;
    p.q = static_cast<const uint8_t*>(a.q);
    p.k = static_cast<const uint8_t*>(a.k);
    p.v = static_cast<const uint8_t*>(a.v);
    p.out = static_cast<uint8_t*>(a.out);
    p.lse = a.lse;
    // scores in base 2: log2(e) / sqrt(D), with the scales of Q and K folded in
    const double qk = a.fp8 ? static_cast<double>(a.q_scale) * a.k_scale : 1.0;
    p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(a.D)) * qk);
    // E4M3 output code = O / o_scale (o_scale is the output's dequantization scale)
    p.out_mul = a.fp8 ? static_cast<float>(static_cast<double>(a.v_scale) / a.o_scale) : 1.f;
    p.after_residual = 0;
    return p;
}

// The prefill kernels follow the schedule build on the same stream as
// programmatic dependent launches: the first one's CTAs may start while the
// build still runs and wait for the build's completion before reading the list;
// the bf16 main variant, launched after the residual variant, starts on the SMs
// that variant leaves and waits for its completion only at its own exit.
cudaError_t launch_prefill(const Args& a, const va::PrefillMaps& maps, const va::PrefillParams& p,
                           int grid, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(va::kPrefillThreads);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (a.fp8) {
        cfg.dynamicSmemBytes = va::PrefillSmem<128, va::ElemE4m3>::kAlloc;
        note_launches(1);
        return cudaLaunchKernelEx(&cfg, va::prefill_fwd_kernel<128, va::ElemE4m3, false>, maps, p);
    }
    // bf16: the residual variant over the list's few-key part first (its CTAs
    // without an item leave at once), then the main variant over the main
    // part as its programmatic dependent, on the SMs the residual one leaves
    va::PrefillParams pm = p;
    pm.after_residual = 1;
    note_launches(2);
    cudaError_t e;
    if (a.D == 64) {
        cfg.dynamicSmemBytes = va::PrefillSmem<64, va::ElemBf16>::kAlloc;
        e = cudaLaunchKernelEx(&cfg, va::prefill_fwd_kernel<64, va::ElemBf16, true>, maps, p);
        if (e != cudaSuccess) return e;
        return cudaLaunchKernelEx(&cfg, va::prefill_fwd_kernel<64, va::ElemBf16, false>, maps, pm);
    }
    cfg.dynamicSmemBytes = va::PrefillSmem<128, va::ElemBf16>::kAlloc;
    e = cudaLaunchKernelEx(&cfg, va::prefill_fwd_kernel<128, va::ElemBf16, true>, maps, p);
    if (e != cudaSuccess) return e;
    return cudaLaunchKernelEx(&cfg, va::prefill_fwd_kernel<128, va::ElemBf16, false>, maps, pm);
}

int run_prefill(const Args& a, const DeviceInfo& dev, cudaStream_t stream) {
    const long long tiles_per_seq = (a.max_q + va::kBlockQ - 1) / va::kBlockQ;
    const long long cap_ll = tiles_per_seq * a.batch;
    if (cap_ll * a.H >= INT_MAX) return fail(VA_ERR_UNSUPPORTED, "too many query tiles x heads");
    const int cap = static_cast<int>(cap_ll);
    int key_slots = 1;
    while (key_slots < cap && key_slots < va::kSortCapacity) key_slots <<= 1;

    const size_t hdr_bytes = 256;
    const size_t list_bytes = static_cast<size_t>(cap) * sizeof(va::TileEntry);
    char* ws = nullptr;
    VA_CUDA(ws_alloc(reinterpret_cast<void**>(&ws), hdr_bytes + 2 * list_bytes, stream));
    auto* hdr = reinterpret_cast<va::SchedHeader*>(ws);
    auto* scratch = reinterpret_cast<va::TileEntry*>(ws + hdr_bytes);
    auto* tiles = reinterpret_cast<va::TileEntry*>(ws + hdr_bytes + list_bytes);

    int rc = VA_OK;
    va::PrefillMaps maps;
    if ((rc = make_prefill_maps(a, &maps)) != VA_OK) {
        cudaFreeAsync(ws, stream);
        return rc;
    }

    note_launches(1);
    va::build_schedule_kernel<<<1, va::kBuildThreads, key_slots * 8, stream>>>(
        a.cu_q, a.cu_k, a.seqused_k, a.batch, a.causal, a.window, a.fp8 ? 0 : 1, cap, key_slots,
        scratch, tiles, hdr);
    cudaError_t be = cudaGetLastError();
    if (be != cudaSuccess) {
        cudaFreeAsync(ws, stream);
        return cuda_fail(be, "schedule build launch");
    }

    va::PrefillParams p = prefill_params(a);
    p.tiles = tiles;
    p.hdr = hdr;
    p.tile_capacity = cap;
    const long long items = cap_ll * a.H;
    const int grid = static_cast<int>(std::min<long long>(dev.num_sms, items));
    cudaError_t le = launch_prefill(a, maps, p, grid, stream);
    cudaFreeAsync(ws, stream);
    if (le != cudaSuccess) return cuda_fail(le, "prefill launch");
    return VA_OK;
}

int run_decode(const Args& a, const DeviceInfo& dev, int split_keys, cudaStream_t stream) {
    if (split_keys != 0 && (split_keys < 32 || split_keys > 65536))
        return fail(VA_ERR_INVALID_ARG, "decode_split_keys must be in [32, 65536] (got %d)", split_keys);
    const int G = a.H / a.H_kv;
    const long long groups = static_cast<long long>(a.H_kv) * ((G + va::kDecodeHeads - 1) / va::kDecodeHeads);
    int chunk = split_keys;
    if (chunk == 0) {
        // fewest splits that still give every SM several units to claim
        const long long want = static_cast<long long>(va::kDecodeUnitsPerSm) * dev.num_sms;
        chunk = va::kDecodeMaxDefaultChunk;
        while (chunk > va::kDecodeMinDefaultChunk &&
               groups * a.batch * ((a.max_k + chunk - 1) / chunk) < want)
            chunk /= 2;
    }
    const int n_split_max = std::max(1, (a.max_k + chunk - 1) / chunk);
    const long long n_units = groups * a.batch * n_split_max;
    if (n_units >= INT_MAX) return fail(VA_ERR_UNSUPPORTED, "decode work units beyond int32");
    const size_t slots = static_cast<size_t>(a.batch) * a.H * n_split_max;
    const size_t hdr = 256;
    const size_t o_bytes = slots * a.D * sizeof(float);
    char* ws = nullptr;
    VA_CUDA(ws_alloc(reinterpret_cast<void**>(&ws), hdr + o_bytes + slots * 4 * sizeof(float), stream));
    cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(int), stream);
    if (e != cudaSuccess) {
        cudaFreeAsync(ws, stream);
        return cuda_fail(e, "cudaMemsetAsync (decode work counter)");
    }
    CUtensorMap tk, tv, tk8, tv8;
    const long long rows_k = std::max(1ll, static_cast<long long>(a.batch) * a.max_k);
    const long long cols_k = static_cast<long long>(a.H_kv) * a.D;
    int rc;
    if ((rc = make_tile_map(&tk, a.k, cols_k, rows_k, va::kDecodeTileKeys)) != VA_OK ||
        (rc = make_tile_map(&tv, a.v, cols_k, rows_k, va::kDecodeTileKeys)) != VA_OK ||
        (rc = make_tile_map(&tk8, a.k, cols_k, rows_k, 8)) != VA_OK ||
        (rc = make_tile_map(&tv8, a.v, cols_k, rows_k, 8)) != VA_OK) {
        cudaFreeAsync(ws, stream);
        return rc;
    }

    va::DecodeParams p;
    p.cu_q = a.cu_q;
    p.cu_k = a.cu_k;
    p.seqused_k = a.seqused_k;
    p.batch = a.batch;
    p.H = a.H;
    p.H_kv = a.H_kv;
    p.causal = a.causal;
    p.window = a.window;
    p.q = static_cast<const __nv_bfloat16*>(a.q);
    p.k = static_cast<const __nv_bfloat16*>(a.k);
    p.v = static_cast<const __nv_bfloat16*>(a.v);
    p.counter = reinterpret_cast<int*>(ws);
    p.part_o = reinterpret_cast<float*>(ws + hdr);
    p.part_ml = reinterpret_cast<float*>(ws + hdr + o_bytes);
    p.n_split_max = n_split_max;
    p.chunk = chunk;
    p.n_units = static_cast<int>(n_units);
    p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(a.D)));
    p.out = static_cast<__nv_bfloat16*>(a.out);
    p.lse = a.lse;
    const int grid = static_cast<int>(std::min<long long>(dev.num_sms, n_units));
    if (a.D == 64) {
        note_launches(2);
        va::decode_stream_kernel<64><<<grid, va::kDecodeThreads, va::DecodeSmem<64>::kAlloc, stream>>>(tk, tv, tk8, tv8, p);
        va::decode_combine_kernel<64><<<a.batch * a.H, 64, 0, stream>>>(p);
    } else {
        note_launches(2);
        va::decode_stream_kernel<128><<<grid, va::kDecodeThreads, va::DecodeSmem<128>::kAlloc, stream>>>(tk, tv, tk8, tv8, p);
        va::decode_combine_kernel<128><<<a.batch * a.H, 128, 0, stream>>>(p);
    }
    cudaError_t le = cudaGetLastError();
    cudaFreeAsync(ws, stream);
    if (le != cudaSuccess) return cuda_fail(le, "decode launch");
    return VA_OK;
}

int forward(const Args& a, int path, int split_keys, cudaStream_t stream) {
    int rc = validate(a);
    if (rc != VA_OK) return rc;
    if (path != VA_PATH_AUTO && path != VA_PATH_PREFILL && path != VA_PATH_DECODE)
        return fail(VA_ERR_INVALID_ARG, "unknown path %d", path);
    if (a.batch == 0 || a.max_q == 0) return VA_OK;
    if (a.fp8) {
        // E4M3 runs on the tile kernel for every query length
        if (path == VA_PATH_DECODE)
            return fail(VA_ERR_UNSUPPORTED, "the decode path takes bf16 inputs only");
        path = VA_PATH_PREFILL;
    }
    if (path == VA_PATH_AUTO) path = a.max_q == 1 ? VA_PATH_DECODE : VA_PATH_PREFILL;
    if (path == VA_PATH_DECODE && a.max_q > 1)
        return fail(VA_ERR_INVALID_ARG, "the decode path needs max_seqlen_q <= 1 (got %d)", a.max_q);
    if (static_cast<long long>(a.batch) * a.H > INT_MAX)
        return fail(VA_ERR_UNSUPPORTED, "batch x num_heads beyond int32");
    int dev;
    DeviceInfo* info;
    if ((rc = device_setup(dev, info)) != VA_OK) return rc;
    return path == VA_PATH_DECODE ? run_decode(a, *info, split_keys, stream) : run_prefill(a, *info, stream);
}

// ---------------------------------------------------------------------------
// Backward pass: dQ per query tile (which also forms Delta = rowsum(dout *
// out)), then dK/dV per key tile (backward_sm100.cuh).

struct BwdArgs {
    Args fwd;  // q, k, v, cu_seqlens, sizes, masks; out = the forward output, lse its logsumexp
    const void* dout;
    void *dq, *dk, *dv;
};

int run_backward(const BwdArgs& g, cudaStream_t stream) {
    const Args& a = g.fwd;
    int rc = validate(a);
    if (rc != VA_OK) return rc;
    const char* names[] = {"dout", "dq", "dk", "dv"};
    const void* ptrs[] = {g.dout, g.dq, g.dk, g.dv};
    if (a.batch > 0 && (a.max_q > 0 || a.max_k > 0)) {
        for (int i = 0; i < 4; ++i) {
            if (!ptrs[i]) return fail(VA_ERR_INVALID_ARG, "%s is NULL", names[i]);
            if (!aligned16(ptrs[i])) return fail(VA_ERR_INVALID_ARG, "%s must be 16-byte aligned", names[i]);
        }
    }
    if (a.batch == 0) return VA_OK;
    // the work lists: one entry per 128-row query tile (dQ) and per 128-key tile (dK/dV)
    const long long cap_q_ll = static_cast<long long>(a.batch) * ((a.max_q + va::kBlockM - 1) / va::kBlockM);
    const long long cap_k_ll = static_cast<long long>(a.batch) * ((a.max_k + va::kBlockN - 1) / va::kBlockN);
    if (cap_q_ll * a.H >= INT_MAX || cap_k_ll * a.H_kv >= INT_MAX)
        return fail(VA_ERR_UNSUPPORTED, "too many tiles x heads for the backward work lists");
    const int cap_q = static_cast<int>(cap_q_ll), cap_k = static_cast<int>(cap_k_ll);
    int dev;
    DeviceInfo* info;
    if ((rc = device_setup(dev, info)) != VA_OK) return rc;
    const long long rows_q = std::max(1ll, static_cast<long long>(a.batch) * a.max_q);
    const long long rows_k = std::max(1ll, static_cast<long long>(a.batch) * a.max_k);
    const long long cols_q = static_cast<long long>(a.H) * a.D;
    const long long cols_k = static_cast<long long>(a.H_kv) * a.D;
    va::BwdMaps maps;
    if ((rc = make_tile_map(&maps.q, a.q, cols_q, rows_q, va::kBlockM)) != VA_OK ||
        (rc = make_tile_map(&maps.dout, g.dout, cols_q, rows_q, va::kBlockM)) != VA_OK ||
        (rc = make_tile_map(&maps.k, a.k, cols_k, rows_k, va::kBlockN)) != VA_OK ||
        (rc = make_tile_map(&maps.v, a.v, cols_k, rows_k, va::kBlockN)) != VA_OK ||
        (rc = make_tile_map(&maps.q8, a.q, cols_q, rows_q, 8)) != VA_OK ||
        (rc = make_tile_map(&maps.dout8, g.dout, cols_q, rows_q, 8)) != VA_OK ||
        (rc = make_tile_map(&maps.k8, a.k, cols_k, rows_k, 8)) != VA_OK ||
        (rc = make_tile_map(&maps.v8, a.v, cols_k, rows_k, 8)) != VA_OK)
        return rc;
    // workspace: {lse * log2(e), Delta} per (head, query row), two list headers,
    // the two lists (each with its sort's second buffer)
    auto up256 = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
    const size_t ri_bytes = up256(static_cast<size_t>(rows_q) * a.H * sizeof(float2));
    const size_t lq_bytes = static_cast<size_t>(cap_q) * sizeof(va::TileEntry);
    const size_t lk_bytes = static_cast<size_t>(cap_k) * sizeof(va::TileEntry);
    char* ws = nullptr;
    VA_CUDA(ws_alloc(reinterpret_cast<void**>(&ws), ri_bytes + 512 + up256(2 * lq_bytes) + 2 * lk_bytes, stream));
    float2* rowinfo = reinterpret_cast<float2*>(ws);
    auto* hdr_q = reinterpret_cast<va::SchedHeader*>(ws + ri_bytes);
    auto* hdr_k = reinterpret_cast<va::SchedHeader*>(ws + ri_bytes + 256);
    auto* scratch_q = reinterpret_cast<va::TileEntry*>(ws + ri_bytes + 512);
    auto* list_q = scratch_q + cap_q;
    auto* scratch_k = reinterpret_cast<va::TileEntry*>(ws + ri_bytes + 512 + up256(2 * lq_bytes));
    auto* list_k = scratch_k + cap_k;
    auto slots = [](int cap) {
        int s = 1;
        while (s < cap && s < va::kSortCapacity) s <<= 1;
        return s;
    };
    if (cap_q > 0)
        note_launches(2);
        va::build_bwd_list_kernel<<<1, va::kBuildThreads, slots(cap_q) * 8, stream>>>(
            a.cu_q, a.cu_k, a.batch, a.causal, a.window, 0, cap_q, slots(cap_q), scratch_q, list_q, hdr_q);
    if (cap_k > 0)
        va::build_bwd_list_kernel<<<1, va::kBuildThreads, slots(cap_k) * 8, stream>>>(
            a.cu_q, a.cu_k, a.batch, a.causal, a.window, 1, cap_k, slots(cap_k), scratch_k, list_k, hdr_k);
    va::BwdParams p;
    p.cu_q = a.cu_q;
    p.cu_k = a.cu_k;
    p.batch = a.batch;
    p.H = a.H;
    p.H_kv = a.H_kv;
    p.causal = a.causal;
    p.window = a.window;
    p.q = static_cast<const uint8_t*>(a.q);
    p.k = static_cast<const uint8_t*>(a.k);
    p.v = static_cast<const uint8_t*>(a.v);
    p.dout = static_cast<const uint8_t*>(g.dout);
    p.out = static_cast<const uint8_t*>(a.out);
    p.lse = a.lse;
    p.rowinfo = rowinfo;
    p.rows_cap = rows_q;
    p.dq = static_cast<uint8_t*>(g.dq);
    p.dk = static_cast<uint8_t*>(g.dk);
    p.dv = static_cast<uint8_t*>(g.dv);
    p.scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(a.D)));
    p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(a.D)));
    p.list_q = list_q;
    p.hdr_q = hdr_q;
    p.cap_q = cap_q;
    p.list_k = list_k;
    p.hdr_k = hdr_k;
    p.cap_k = cap_k;
    // persistent grids, one CTA per SM (fewer when there are fewer items);
    // dQ first: it forms Delta for every query row that sees a key, which the
    // dK/dV kernel reads
    const int grid_q = static_cast<int>(std::min<long long>(info->num_sms, cap_q_ll * a.H));
    const int grid_kv = static_cast<int>(std::min<long long>(info->num_sms, cap_k_ll * a.H_kv));
    note_launches((grid_q > 0) + (grid_kv > 0));
    if (a.D == 64) {
        if (grid_q > 0) va::bwd_dq_kernel<64><<<grid_q, va::kBwdThreads, va::BwdSmem<64, true>::kAlloc, stream>>>(maps, p);
        if (grid_kv > 0)
            va::bwd_dkdv_kernel<64><<<grid_kv, va::kBwdThreads, va::BwdSmem<64, false>::kAlloc, stream>>>(maps, p);
    } else {
        if (grid_q > 0)
            va::bwd_dq_kernel<128><<<grid_q, va::kBwdThreads, va::BwdSmem<128, true>::kAlloc, stream>>>(maps, p);
        if (grid_kv > 0)
            va::bwd_dkdv_kernel<128><<<grid_kv, va::kBwdThreads, va::BwdSmem<128, false>::kAlloc, stream>>>(maps, p);
    }
    cudaError_t le = cudaGetLastError();
    cudaFreeAsync(ws, stream);
    if (le != cudaSuccess) return cuda_fail(le, "backward launch");
    return VA_OK;
}

// ---------------------------------------------------------------------------
// Entry point without allocation.  Some callers must not reach any device
// allocator: code running inside a framework or serving runtime that owns all
// device memory through its own allocator, or a latency-critical loop that may
// not call cudaMalloc or a stream-ordered allocator.  For them the prefill
// path's workspace (the work-list header and two copies of the query-block
// list) lives in a fixed static device array instead.

constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;  // 1 MiB per device
constexpr size_t kNoAllocHeaderBytes = 256;
// query blocks the array can describe: header + scratch list + sorted list
constexpr long long kNoAllocMaxBlocks =
    static_cast<long long>((kNoAllocScratchBytes - kNoAllocHeaderBytes) / (2 * sizeof(va::TileEntry)));

struct NoAllocState {
    bool ready = false;
    int num_sms = 0;
    unsigned char* scratch = nullptr;  // device address of g_noalloc_scratch on this device
};
NoAllocState g_noalloc[kMaxDevices];

}  // namespace

// One copy per device that loads the library, held until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

// Once per device, with that device current: kernel attributes, the tensor-map
// encoder and the device address of the static scratch array (in host code the
// array's name is only a stand-in, not an address a kernel may be given).
int noalloc_setup(NoAllocState*& st) {
    int dev = 0;
    VA_CUDA(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) return fail(VA_ERR_UNSUPPORTED, "device ordinal %d", dev);
    std::lock_guard<std::mutex> lock(g_dev_mu);
    st = &g_noalloc[dev];
    if (st->ready) return VA_OK;
    cudaDeviceProp prop;
    VA_CUDA(cudaGetDeviceProperties(&prop, dev));
    if (prop.major != 10)
        return fail(VA_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a",
                    dev, prop.major, prop.minor);
    if (!g_encode) {
        cudaDriverEntryPointQueryResult q;
        void* fn = nullptr;
        VA_CUDA(cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q));
        if (q != cudaDriverEntryPointSuccess || !fn)
            return fail(VA_ERR_CUDA, "cuTensorMapEncodeTiled entry point not found");
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    if (set_prefill_attributes() != VA_OK) return VA_ERR_CUDA;
    VA_CUDA(cudaFuncSetAttribute(va::build_schedule_kernel,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 va::kSortCapacity * 8));
    void* addr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&addr, g_noalloc_scratch);
    if (e != cudaSuccess || addr == nullptr)
        return cuda_fail(e == cudaSuccess ? cudaErrorInvalidSymbol : e,
                         "cudaGetSymbolAddress(g_noalloc_scratch)");
    st->scratch = static_cast<unsigned char*>(addr);
    st->num_sms = prop.multiProcessorCount;
    st->ready = true;
    return VA_OK;
}

int run_prefill_noalloc(const Args& a, cudaStream_t stream) {
    const long long blocks = static_cast<long long>(a.batch) * ((a.max_q + va::kBlockQ - 1) / va::kBlockQ);
    if (blocks > kNoAllocMaxBlocks)
        return fail(VA_ERR_UNSUPPORTED,
                    "batch x ceil(max_seqlen_q / %d) = %lld query blocks exceeds the %lld that the "
                    "%zu-byte static scratch holds; use varlen_attention_fwd",
                    va::kBlockQ, blocks, kNoAllocMaxBlocks, kNoAllocScratchBytes);
    if (blocks * a.H >= INT_MAX) return fail(VA_ERR_UNSUPPORTED, "too many query blocks x heads");
    NoAllocState* st = nullptr;
    int rc = noalloc_setup(st);
    if (rc != VA_OK) return rc;
    const int cap = static_cast<int>(blocks);
    int key_slots = 1;
    while (key_slots < cap && key_slots < va::kSortCapacity) key_slots <<= 1;
    const size_t list_bytes = static_cast<size_t>(cap) * sizeof(va::TileEntry);
    auto* hdr = reinterpret_cast<va::SchedHeader*>(st->scratch);
    auto* scratch = reinterpret_cast<va::TileEntry*>(st->scratch + kNoAllocHeaderBytes);
    auto* tiles = reinterpret_cast<va::TileEntry*>(st->scratch + kNoAllocHeaderBytes + list_bytes);

    va::PrefillMaps maps;
    if ((rc = make_prefill_maps(a, &maps)) != VA_OK) return rc;
    // the builder rewrites the whole header (count and work counter) and every
    // list entry it hands out, so nothing left by the previous call is read
    note_launches(1);
    va::build_schedule_kernel<<<1, va::kBuildThreads, key_slots * 8, stream>>>(
        a.cu_q, a.cu_k, a.seqused_k, a.batch, a.causal, a.window, a.fp8 ? 0 : 1, cap, key_slots,
        scratch, tiles, hdr);
    cudaError_t be = cudaGetLastError();
    if (be != cudaSuccess) return cuda_fail(be, "schedule build launch");

    va::PrefillParams p = prefill_params(a);
    p.tiles = tiles;
    p.hdr = hdr;
    p.tile_capacity = cap;
    const int grid = static_cast<int>(std::min<long long>(st->num_sms, blocks * a.H));
    cudaError_t le = launch_prefill(a, maps, p, grid, stream);
    if (le != cudaSuccess) return cuda_fail(le, "prefill launch");
    return VA_OK;
}

// One chunk of the host-buffer entry point's pipeline: the packed query rows
// [q0, q1) and, for its kernels, the keys from packed row k_base on.
struct HostChunk {
    bool piece;           // part of one sequence (b0) rather than whole sequences [b0, b1)
    int b0, b1;
    long long q0, q1;     // packed query rows
    long long k_base;     // packed key row of the chunk's key 0
    long long k_len;      // a piece's key count (a group's come from cu_seqlens)
    long long kc0, kc1;   // packed key rows this chunk copies in (none an earlier chunk brought)
};

// Plan of the host-buffer pipeline.  Sequences are grouped whole until a
// group holds about 1/kHostChunks of the query rows; a sequence longer than
// that is cut into pieces of whole 256-row query blocks, each with the keys
// its rows can see: the keys up to its last row's diagonal (causal, or a
// window, which also bounds the keys from below, rounded down to a 128-key
// tile) or all of the sequence's keys (neither).  The piece then computes
// exactly what the whole sequence's launch computes for those rows: the same
// query blocks, the same key tiles in the same order, the same masks (its
// bottom-right diagonal offset is the sequence's, shifted by the keys left
// out below), so the results are bit-identical.
std::vector<HostChunk> plan_host_chunks(const int32_t* cu_q, const int32_t* cu_k, int batch, bool causal,
                                        int window, size_t input_bytes) {
    std::vector<HostChunk> out;
    const long long T_q = cu_q[batch];
    if (input_bytes < kHostChunkMinBytes || T_q == 0) {
        out.push_back(HostChunk{false, 0, batch, 0, T_q, 0, 0, 0, cu_k[batch]});
        return out;
    }
    const long long blk = va::kBlockQ;
    const long long rows = std::max<long long>(kHostChunkMinRows,
                                               (T_q + kHostChunks - 1) / kHostChunks + blk - 1) / blk * blk;
    int g0 = 0;  // first sequence of the open group
    auto close_group = [&](int b1) {
        if (b1 > g0)
            out.push_back(HostChunk{false, g0, b1, cu_q[g0], cu_q[b1], cu_k[g0], 0, cu_k[g0], cu_k[b1]});
        g0 = b1;
    };
    for (int b = 0; b < batch; ++b) {
        const long long L_q = cu_q[b + 1] - cu_q[b], L_k = cu_k[b + 1] - cu_k[b];
        if (L_q <= rows) {
            if (cu_q[b + 1] - cu_q[g0] >= rows) close_group(b + 1);
            continue;
        }
        close_group(b);
        const long long delta = L_k - L_q;
        const bool banded = causal || window > 0;
        long long copied = 0;  // keys of this sequence already copied in
        for (long long r0 = 0; r0 < L_q; r0 += rows) {
            const long long r1 = std::min(L_q, r0 + rows);
            long long k_lo = 0, k_hi = L_k;
            if (banded) {
                k_hi = std::min(L_k, std::max(0ll, r1 + delta));
                if (window > 0) k_lo = std::max(0ll, r0 + delta - window + 1) / va::kBlockN * va::kBlockN;
                k_lo = std::min(k_lo, k_hi);
            }
            const long long c1 = std::max(copied, k_hi);
            out.push_back(HostChunk{true, b, b + 1, cu_q[b] + r0, cu_q[b] + r1, cu_k[b] + k_lo, k_hi - k_lo,
                                    cu_k[b] + copied, cu_k[b] + c1});
            copied = c1;
        }
        g0 = b + 1;
    }
    close_group(batch);
    return out;
}

}  // namespace

extern "C" {

int varlen_attention_fwd(const void* q, const void* k, const void* v, const int32_t* cu_seqlens_q,
                         const int32_t* cu_seqlens_k, int batch, int num_heads, int num_kv_heads,
                         int max_seqlen_q, int max_seqlen_k, int head_dim, int causal, int window,
                         void* out, float* lse, void* stream) {
    g_last_error[0] = 0;
    Args a{q, k, v, cu_seqlens_q, cu_seqlens_k, batch, num_heads, num_kv_heads, max_seqlen_q,
           max_seqlen_k, head_dim, causal ? 1 : 0, window, out, lse};
    return forward(a, VA_PATH_AUTO, 0, static_cast<cudaStream_t>(stream));
}

int varlen_attention_fwd_fp8(const void* q, const void* k, const void* v,
                             const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int batch,
                             int num_heads, int num_kv_heads, int max_seqlen_q, int max_seqlen_k,
                             int head_dim, int causal, int window, float q_scale, float k_scale,
                             float v_scale, float o_scale, void* out, float* lse, void* stream) {
    g_last_error[0] = 0;
    Args a{q, k, v, cu_seqlens_q, cu_seqlens_k, batch, num_heads, num_kv_heads, max_seqlen_q,
           max_seqlen_k, head_dim, causal ? 1 : 0, window, out, lse};
    a.fp8 = 1;
    a.q_scale = q_scale;
    a.k_scale = k_scale;
    a.v_scale = v_scale;
    a.o_scale = o_scale;
    return forward(a, VA_PATH_AUTO, 0, static_cast<cudaStream_t>(stream));
}

int varlen_attention_bwd(const void* dout, const void* q, const void* k, const void* v,
                         const void* out, const float* lse, const int32_t* cu_seqlens_q,
                         const int32_t* cu_seqlens_k, int batch, int num_heads, int num_kv_heads,
                         int max_seqlen_q, int max_seqlen_k, int head_dim, int causal, int window,
                         void* dq, void* dk, void* dv, void* stream) {
    g_last_error[0] = 0;
    BwdArgs g{Args{q, k, v, cu_seqlens_q, cu_seqlens_k, batch, num_heads, num_kv_heads,
                   max_seqlen_q, max_seqlen_k, head_dim, causal ? 1 : 0, window,
                   const_cast<void*>(out), const_cast<float*>(lse)},
              dout, dq, dk, dv};
    return run_backward(g, static_cast<cudaStream_t>(stream));
}

int varlen_attention_fwd_kvcache(const void* q, const void* k, const void* v,
                                 const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                                 const int32_t* seqused_k, int batch, int num_heads,
                                 int num_kv_heads, int max_seqlen_q, int max_seqlen_k, int head_dim,
                                 int causal, int window, void* out, float* lse, void* stream) {
    g_last_error[0] = 0;
    if (!seqused_k) return fail(VA_ERR_INVALID_ARG, "seqused_k is NULL (use varlen_attention_fwd)");
    Args a{q, k, v, cu_seqlens_q, cu_seqlens_k, batch, num_heads, num_kv_heads, max_seqlen_q,
           max_seqlen_k, head_dim, causal ? 1 : 0, window, out, lse};
    a.seqused_k = seqused_k;
    return forward(a, VA_PATH_AUTO, 0, static_cast<cudaStream_t>(stream));
}

int varlen_attention_fwd_ex(const void* q, const void* k, const void* v,
                            const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int batch,
                            int num_heads, int num_kv_heads, int max_seqlen_q, int max_seqlen_k,
                            int head_dim, int causal, int window, void* out, float* lse, int path,
                            int decode_split_keys, void* stream) {
    g_last_error[0] = 0;
    Args a{q, k, v, cu_seqlens_q, cu_seqlens_k, batch, num_heads, num_kv_heads, max_seqlen_q,
           max_seqlen_k, head_dim, causal ? 1 : 0, window, out, lse};
    return forward(a, path, decode_split_keys, static_cast<cudaStream_t>(stream));
}

int varlen_attention_fwd_host(const void* q, const void* k, const void* v,
                              const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int batch,
                              int num_heads, int num_kv_heads, int max_seqlen_q, int max_seqlen_k,
                              int head_dim, int causal, int window, void* out, float* lse,
                              void* stream_) {
    g_last_error[0] = 0;
    Args a{q, k, v, cu_seqlens_q, cu_seqlens_k, batch, num_heads, num_kv_heads, max_seqlen_q,
           max_seqlen_k, head_dim, causal ? 1 : 0, window, out, lse};
    int rc = validate(a);
    if (rc != VA_OK) return rc;
    if (batch == 0 || max_seqlen_q == 0) return VA_OK;
    // The host arrays size every copy and every chunk below: check them before
    // any device work (a decreasing entry would give negative offsets).
    if ((rc = check_cu_seqlens_host(cu_seqlens_q, batch, max_seqlen_q, -1, "cu_seqlens_q")) != VA_OK ||
        (rc = check_cu_seqlens_host(cu_seqlens_k, batch, max_seqlen_k, -1, "cu_seqlens_k")) != VA_OK)
        return rc;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    int dev;
    DeviceInfo* info;
    if ((rc = device_setup(dev, info)) != VA_OK) return rc;
    const long long T_q = cu_seqlens_q[batch], T_k = cu_seqlens_k[batch];
    const size_t q_row = static_cast<size_t>(num_heads) * head_dim * 2;
    const size_t k_row = static_cast<size_t>(num_kv_heads) * head_dim * 2;
    const size_t l_row = static_cast<size_t>(num_heads) * 4;
    const size_t qb = static_cast<size_t>(T_q) * q_row, kb = static_cast<size_t>(T_k) * k_row;
    const size_t ob = qb, lb = static_cast<size_t>(T_q) * l_row;

    // Chunks in packed query order: groups of whole sequences, and pieces of
    // one long sequence (whole 256-row query blocks with the keys they can
    // see).  Chunk i's kernels run while chunk i + 1 is copied in and chunk
    // i - 1 is copied out (the two directions on separate streams and copy
    // engines).
    const std::vector<HostChunk> chunks =
        plan_host_chunks(cu_seqlens_q, cu_seqlens_k, batch, causal != 0, window, qb + 2 * kb);
    const int n = static_cast<int>(chunks.size());
    // per chunk, cu_seqlens rebased to the chunk's first query row and first key
    std::vector<int32_t> cu_h;
    std::vector<size_t> cu_off(n);
    for (int c = 0; c < n; ++c) {
        const HostChunk& h = chunks[c];
        cu_off[c] = cu_h.size();
        if (h.piece) {
            cu_h.insert(cu_h.end(), {0, static_cast<int32_t>(h.q1 - h.q0)});
            cu_h.insert(cu_h.end(), {0, static_cast<int32_t>(h.k_len)});
        } else {
            for (int b = h.b0; b <= h.b1; ++b) cu_h.push_back(cu_seqlens_q[b] - cu_seqlens_q[h.b0]);
            for (int b = h.b0; b <= h.b1; ++b) cu_h.push_back(cu_seqlens_k[b] - cu_seqlens_k[h.b0]);
        }
    }
    const size_t cb = cu_h.size() * sizeof(int32_t);

    auto up256 = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
    const size_t total = up256(qb) + 2 * up256(kb) + up256(cb) + up256(ob) + up256(lb);
    cudaStream_t s_in = stream, s_out = stream;
    if (n > 1) {
        std::lock_guard<std::mutex> lock(g_dev_mu);
        if (!info->copy_in) VA_CUDA(cudaStreamCreateWithFlags(&info->copy_in, cudaStreamNonBlocking));
        if (!info->copy_out) VA_CUDA(cudaStreamCreateWithFlags(&info->copy_out, cudaStreamNonBlocking));
        s_in = info->copy_in;
        s_out = info->copy_out;
    }
    char* ws = nullptr;
    VA_CUDA(ws_alloc(reinterpret_cast<void**>(&ws), total, stream));
    char* p = ws;
    char* dq = p; p += up256(qb);
    char* dk = p; p += up256(kb);
    char* dv = p; p += up256(kb);
    int32_t* dcu = reinterpret_cast<int32_t*>(p); p += up256(cb);
    char* dout = p; p += up256(ob);
    float* dlse = reinterpret_cast<float*>(p);

    // events: [0] workspace ready, [1 .. n] chunk c copied in, [n + 1 .. 2n]
    // chunk c computed, [2n + 1] / [2n + 2] the copy streams drained
    std::vector<cudaEvent_t> ev;
    cudaError_t e = cudaSuccess;
    if (n > 1) {
        ev.resize(2 * n + 3, nullptr);
        for (auto& x : ev)
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&x, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventRecord(ev[0], stream);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(s_in, ev[0], 0);
    }
    // every host-to-device copy, chunk after chunk, on the input stream: the
    // chunk's query rows and the key rows it needs that no earlier chunk
    // brought (a chunk's event so also covers every earlier copy)
    if (e == cudaSuccess && cb) e = cudaMemcpyAsync(dcu, cu_h.data(), cb, cudaMemcpyHostToDevice, s_in);
    for (int c = 0; c < n && e == cudaSuccess; ++c) {
        const HostChunk& h = chunks[c];
        if (h.q1 > h.q0)
            e = cudaMemcpyAsync(dq + h.q0 * q_row, static_cast<const char*>(q) + h.q0 * q_row,
                                (h.q1 - h.q0) * q_row, cudaMemcpyHostToDevice, s_in);
        if (e == cudaSuccess && h.kc1 > h.kc0)
            e = cudaMemcpyAsync(dk + h.kc0 * k_row, static_cast<const char*>(k) + h.kc0 * k_row,
                                (h.kc1 - h.kc0) * k_row, cudaMemcpyHostToDevice, s_in);
        if (e == cudaSuccess && h.kc1 > h.kc0)
            e = cudaMemcpyAsync(dv + h.kc0 * k_row, static_cast<const char*>(v) + h.kc0 * k_row,
                                (h.kc1 - h.kc0) * k_row, cudaMemcpyHostToDevice, s_in);
        if (e == cudaSuccess && n > 1) e = cudaEventRecord(ev[1 + c], s_in);
    }
    // chunk by chunk: its kernels on the caller's stream, then its results
    // back on the output stream
    for (int c = 0; c < n && e == cudaSuccess && rc == VA_OK; ++c) {
        const HostChunk& h = chunks[c];
        if (n > 1) e = cudaStreamWaitEvent(stream, ev[1 + c], 0);
        if (e != cudaSuccess) break;
        const int nb = h.piece ? 1 : h.b1 - h.b0;
        Args d{dq + h.q0 * q_row, dk + h.k_base * k_row, dv + h.k_base * k_row, dcu + cu_off[c],
               dcu + cu_off[c] + nb + 1, nb, num_heads, num_kv_heads, max_seqlen_q, max_seqlen_k,
               head_dim, causal ? 1 : 0, window, dout + h.q0 * q_row, dlse + h.q0 * num_heads};
        rc = forward(d, VA_PATH_AUTO, 0, stream);
        if (rc != VA_OK) break;
        if (n > 1) {
            e = cudaEventRecord(ev[1 + n + c], stream);
            if (e == cudaSuccess) e = cudaStreamWaitEvent(s_out, ev[1 + n + c], 0);
        }
        if (e == cudaSuccess && h.q1 > h.q0)
            e = cudaMemcpyAsync(static_cast<char*>(out) + h.q0 * q_row, dout + h.q0 * q_row,
                                (h.q1 - h.q0) * q_row, cudaMemcpyDeviceToHost, s_out);
        if (e == cudaSuccess && h.q1 > h.q0)
            e = cudaMemcpyAsync(reinterpret_cast<char*>(lse) + h.q0 * l_row,
                                reinterpret_cast<char*>(dlse) + h.q0 * l_row, (h.q1 - h.q0) * l_row,
                                cudaMemcpyDeviceToHost, s_out);
    }
    // the caller's stream waits for both copy streams (also after an error,
    // so that nothing still reads the workspace when it is freed)
    if (n > 1) {
        cudaError_t w = (ev[2 * n + 1] && ev[2 * n + 2]) ? cudaSuccess : cudaErrorInvalidResourceHandle;
        if (w == cudaSuccess) w = cudaEventRecord(ev[2 * n + 1], s_in);
        if (w == cudaSuccess) w = cudaStreamWaitEvent(stream, ev[2 * n + 1], 0);
        if (w == cudaSuccess) w = cudaEventRecord(ev[2 * n + 2], s_out);
        if (w == cudaSuccess) w = cudaStreamWaitEvent(stream, ev[2 * n + 2], 0);
        if (w != cudaSuccess) {
            // could not order the copy streams before the free: drain them
            cudaStreamSynchronize(s_in);
            cudaStreamSynchronize(s_out);
        }
    }
    cudaFreeAsync(ws, stream);
    cudaError_t se = cudaStreamSynchronize(stream);
    for (auto& x : ev)
        if (x) cudaEventDestroy(x);
    if (rc != VA_OK) return rc;
    if (e != cudaSuccess) return cuda_fail(e, "host-buffer copies");
    if (se != cudaSuccess) return cuda_fail(se, "cudaStreamSynchronize");
    return VA_OK;
}

int varlen_attention_host_chunks(const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int batch,
                                 int causal, int window, long long input_bytes, long long* chunks,
                                 int capacity, int* n_chunks) {
    g_last_error[0] = 0;
    if (!cu_seqlens_q || !cu_seqlens_k || !n_chunks)
        return fail(VA_ERR_INVALID_ARG, "cu_seqlens_q, cu_seqlens_k and n_chunks must not be NULL");
    if (batch < 0) return fail(VA_ERR_INVALID_ARG, "batch must be >= 0 (got %d)", batch);
    if (window < 0) return fail(VA_ERR_INVALID_ARG, "window must be >= 0 (got %d)", window);
    int rc;
    if ((rc = check_cu_seqlens_host(cu_seqlens_q, batch, INT_MAX, -1, "cu_seqlens_q")) != VA_OK ||
        (rc = check_cu_seqlens_host(cu_seqlens_k, batch, INT_MAX, -1, "cu_seqlens_k")) != VA_OK)
        return rc;
    const std::vector<HostChunk> plan = plan_host_chunks(
        cu_seqlens_q, cu_seqlens_k, batch, causal != 0, window, static_cast<size_t>(std::max(0ll, input_bytes)));
    *n_chunks = static_cast<int>(plan.size());
    if (static_cast<int>(plan.size()) > capacity || (!chunks && !plan.empty()))
        return fail(VA_ERR_INVALID_ARG, "capacity %d below the %zu chunks of the plan", capacity, plan.size());
    for (size_t c = 0; c < plan.size(); ++c) {
        const HostChunk& h = plan[c];
        const long long f[9] = {h.piece ? 1 : 0, h.b0, h.b1, h.q0, h.q1, h.k_base, h.k_len, h.kc0, h.kc1};
        std::copy(f, f + 9, chunks + 9 * c);
    }
    return VA_OK;
}

int varlen_attention_schedule(const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int batch,
                              int max_seqlen_q, int causal, int window, int32_t* tiles,
                              int32_t* n_tiles, int capacity, void* stream_) {
    g_last_error[0] = 0;
    if (batch < 1) return fail(VA_ERR_INVALID_ARG, "batch must be >= 1 (got %d)", batch);
    if (!cu_seqlens_q || !cu_seqlens_k || !tiles || !n_tiles)
        return fail(VA_ERR_INVALID_ARG, "NULL pointer argument");
    if (capacity < 1 || window < 0 || max_seqlen_q < 0)
        return fail(VA_ERR_INVALID_ARG, "capacity must be >= 1, window and max_seqlen_q >= 0");
    if (reinterpret_cast<uintptr_t>(tiles) & 15u) return fail(VA_ERR_INVALID_ARG, "tiles must be 16-byte aligned");
    int dev;
    DeviceInfo* info;
    int rc = device_setup(dev, info);
    if (rc != VA_OK) return rc;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    int key_slots = 1;
    while (key_slots < capacity && key_slots < va::kSortCapacity) key_slots <<= 1;
    char* ws = nullptr;
    const size_t list_bytes = static_cast<size_t>(capacity) * sizeof(va::TileEntry);
    VA_CUDA(ws_alloc(reinterpret_cast<void**>(&ws), 256 + list_bytes, stream));
    auto* hdr = reinterpret_cast<va::SchedHeader*>(ws);
    note_launches(1);
    va::build_schedule_kernel<<<1, va::kBuildThreads, key_slots * 8, stream>>>(
        cu_seqlens_q, cu_seqlens_k, nullptr, batch, causal ? 1 : 0, window, 1, capacity, key_slots,
        reinterpret_cast<va::TileEntry*>(ws + 256), reinterpret_cast<va::TileEntry*>(tiles), hdr);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(n_tiles, &hdr->n_tiles, sizeof(int32_t), cudaMemcpyDeviceToDevice, stream);
    cudaFreeAsync(ws, stream);
    if (e != cudaSuccess) return cuda_fail(e, "schedule build");
    return VA_OK;
}

int varlen_attention_validate_cu_seqlens(const int32_t* cu_seqlens, int batch, int max_seqlen,
                                         int total, int on_device, void* stream_) {
    g_last_error[0] = 0;
    if (!cu_seqlens) return fail(VA_ERR_INVALID_ARG, "cu_seqlens is NULL");
    if (batch < 0) return fail(VA_ERR_INVALID_ARG, "batch must be >= 0 (got %d)", batch);
    if (max_seqlen < 0) return fail(VA_ERR_INVALID_ARG, "max_seqlen must be >= 0 (got %d)", max_seqlen);
    std::vector<int32_t> host;
    const int32_t* c = cu_seqlens;
    if (on_device) {
        host.resize(static_cast<size_t>(batch) + 1);
        cudaStream_t stream = static_cast<cudaStream_t>(stream_);
        VA_CUDA(cudaMemcpyAsync(host.data(), cu_seqlens, host.size() * sizeof(int32_t),
                                cudaMemcpyDeviceToHost, stream));
        VA_CUDA(cudaStreamSynchronize(stream));
        c = host.data();
    }
    return check_cu_seqlens_host(c, batch, max_seqlen, total, "cu_seqlens");
}

int varlen_attention_device_status(unsigned* status, int clear) {
    g_last_error[0] = 0;
    if (!status) return fail(VA_ERR_INVALID_ARG, "status is NULL");
    VA_CUDA(cudaDeviceSynchronize());
    VA_CUDA(cudaMemcpyFromSymbol(status, va::g_va_status, sizeof(unsigned)));
    if (clear) {
        const unsigned zero = 0;
        VA_CUDA(cudaMemcpyToSymbol(va::g_va_status, &zero, sizeof(unsigned)));
    }
    return VA_OK;
}

int varlen_attention_sync_status(void* stream_, unsigned* status, int clear) {
    g_last_error[0] = 0;
    if (!status) return fail(VA_ERR_INVALID_ARG, "status is NULL");
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    unsigned word = 0;
    VA_CUDA(cudaMemcpyFromSymbolAsync(&word, va::g_va_status, sizeof(unsigned), 0,
                                      cudaMemcpyDeviceToHost, stream));
    if (clear) {
        // after the copy in the same stream's order
        void* addr = nullptr;
        VA_CUDA(cudaGetSymbolAddress(&addr, va::g_va_status));
        VA_CUDA(cudaMemsetAsync(addr, 0, sizeof(unsigned), stream));
    }
    VA_CUDA(cudaStreamSynchronize(stream));
    *status = word;
    if (word & va::kStatusWaitTimeout)
        return fail(VA_ERR_DEVICE_TIMEOUT, "a bounded wait inside a kernel gave up (status 0x%x)", word);
    if (word & va::kStatusSmemAlign)
        return fail(VA_ERR_CUDA, "a kernel's dynamic shared memory was not 1024-byte aligned; it did nothing "
                                 "(status 0x%x)", word);
    if (word & va::kStatusScheduleOverflow)
        return fail(VA_ERR_INVALID_ARG,
                    "more query blocks than max_seqlen_q allows for: a query length exceeds "
                    "max_seqlen_q (status 0x%x)", word);
    return VA_OK;
}

int varlen_attention_fwd_noalloc(const void* q, const void* k, const void* v,
                                 const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int batch,
                                 int num_heads, int num_kv_heads, int max_seqlen_q, int max_seqlen_k,
                                 int head_dim, int causal, int window, void* out, float* lse,
                                 void* stream) {
    g_last_error[0] = 0;
    Args a{q, k, v, cu_seqlens_q, cu_seqlens_k, batch, num_heads, num_kv_heads, max_seqlen_q,
           max_seqlen_k, head_dim, causal ? 1 : 0, window, out, lse};
    int rc = validate(a);
    if (rc != VA_OK) return rc;
    if (batch == 0 || max_seqlen_q == 0) return VA_OK;
    return run_prefill_noalloc(a, static_cast<cudaStream_t>(stream));
}

int varlen_attention_selftest_wait_timeout(int32_t* gave_up, void* stream) {
    g_last_error[0] = 0;
    if (!gave_up) return fail(VA_ERR_INVALID_ARG, "gave_up is NULL");
    note_launches(1);
    va::wait_timeout_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(gave_up);
    VA_CUDA(cudaGetLastError());
    return VA_OK;
}

const char* varlen_attention_last_error(void) { return g_last_error; }

int varlen_attention_version(void) { return 100; }

unsigned long long varlen_attention_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
