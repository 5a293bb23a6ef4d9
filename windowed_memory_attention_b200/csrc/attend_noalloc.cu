// GCA attention over caller-owned pages, with no device allocation.
//
// Why this exists: some callers of the library must not call cudaMalloc.  A
// host framework with its own caching allocator (PyTorch, a serving engine)
// owns the device memory and would see a private cudaMalloc as memory it can
// neither account for nor reuse; a real-time robot loop cannot afford a call
// that may synchronise the device or take an unbounded time.  Such a caller
// keeps the K/V pools in its own memory and calls gca_attend_pages_noalloc,
// which launches the same tcgen05 attention kernel as gca_attend but puts its
// split-KV partial results, their counters (and a device copy of the walk list) in one
// file-scope __device__ array instead of cache-owned scratch.
//
// The array is gca_noalloc_scratch, kNoallocScratchBytes = 18 MiB, resident
// on every GPU that loads libgca.so until the process exits.  Host code must
// not use its name as an address: the first call on a device, with that device
// current, asks the runtime for its device address (cudaGetSymbolAddress) and
// caches it.  That first call should therefore happen before any stream
// capture.  Every call shares the array and it keeps the last call's contents;
// nothing in it needs to start at zero (each partial is written before it is
// read within one call).  Two calls whose GPU work overlaps (different
// streams, or different devices' work is fine) race on the array.
#include <algorithm>
#include <atomic>
#include <mutex>

#include "../../include/gca.h"
#include "gca_internal.h"

namespace {

constexpr int kNoallocMaxWalk = 32768;       // walk-list entries per call
constexpr int kNoallocMaxSlots = 512;        // 128-row partial tiles per call
constexpr size_t kWalkRawBytes = (size_t)kNoallocMaxWalk * sizeof(gca_page_entry_t);
constexpr size_t kWalkBytes = (size_t)kNoallocMaxWalk * sizeof(int4);
constexpr size_t kLseBytes = (size_t)kNoallocMaxSlots * 128 * sizeof(float);
constexpr size_t kPartialBytes = (size_t)kNoallocMaxSlots * 128 * gca::kHeadDim * sizeof(float);
constexpr size_t kStatusBytes = 256;
constexpr size_t kCountBytes = (size_t)kNoallocMaxSlots * sizeof(unsigned long long);   // split-head counters
constexpr size_t kNoallocScratchBytes =
    kStatusBytes + kCountBytes + kWalkRawBytes + kWalkBytes + kLseBytes + kPartialBytes;
static_assert(kNoallocScratchBytes <= (size_t)18 << 20, "scratch stays modest");

}  // namespace

static __device__ __align__(256) unsigned char gca_noalloc_scratch[kNoallocScratchBytes];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {};

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
typedef CUresult (*AddressRangeFn)(CUdeviceptr*, size_t*, CUdeviceptr);
EncodeTiledFn g_encode = nullptr;
AddressRangeFn g_range = nullptr;
std::atomic<unsigned int> g_epoch{0};   // launch epochs of the split-head counters

// Device address of the scratch array on the current device, looked up once
// per device.
unsigned char* scratch_address(int dev) {
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (dev < 0 || dev >= kMaxDevices) return nullptr;
    if (!g_scratch_addr[dev]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, gca_noalloc_scratch) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        g_scratch_addr[dev] = ptr;
    }
    if (!g_encode || !g_range) {
        void* fn = nullptr;
        void* fr = nullptr;
        cudaDriverEntryPointQueryResult q{}, qr{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess || !fn ||
            cudaGetDriverEntryPoint("cuMemGetAddressRange", &fr, cudaEnableDefault, &qr) != cudaSuccess || !fr) {
            cudaGetLastError();
            return nullptr;
        }
        g_encode = (EncodeTiledFn)fn;
        g_range = (AddressRangeFn)fr;
    }
    return static_cast<unsigned char*>(g_scratch_addr[dev]);
}

// public walk-list entries -> the kernel's int4 form {page, n_valid, first, frame or -1}
__global__ void walk_to_int4(const gca_page_entry_t* in, int4* out, int n) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) {
        const gca_page_entry_t e = in[i];
        out[i] = make_int4(e.page_id, e.n_valid, e.first, e.kind == GCA_PAGE_IMAGE ? e.frame : -1);
    }
}

bool is_device_ptr(const void* ptr) {
    cudaPointerAttributes a{};
    if (cudaPointerGetAttributes(&a, ptr) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged;
}

// True when [ptr, ptr + bytes) lies inside the device allocation that holds
// ptr (for memory from a caching allocator: inside the block it carved ptr
// from), so that no kernel of this call reads or writes past it.
bool fits_allocation(const void* ptr, size_t bytes) {
    CUdeviceptr base = 0;
    size_t size = 0;
    if (!g_range || g_range(&base, &size, (CUdeviceptr)ptr) != CUDA_SUCCESS) return false;
    const size_t off = (size_t)((CUdeviceptr)ptr - base);
    return off <= size && bytes <= size - off;
}

}  // namespace

extern "C" int gca_attend_pages_noalloc(const void* k_pool, const void* v_pool, int32_t num_layers,
                                        int32_t num_pages, int32_t num_heads, int32_t page_size,
                                        int32_t layer, const gca_page_entry_t* walk, int32_t nwalk,
                                        const void* q, int32_t num_query_frames,
                                        int32_t tokens_per_frame, int32_t first_query_frame,
                                        int32_t num_anchor, int32_t window, int32_t summary_tokens,
                                        int32_t anchor_block, float softmax_scale, void* out,
                                        float* lse, int32_t* status, void* stream) {
    if (!k_pool || !v_pool || !walk || !q || !out) return GCA_ERR_INVALID_ARG;
    if (num_layers < 1 || num_pages < 1 || num_heads < 1 || layer < 0 || layer >= num_layers ||
        nwalk < 1 || num_query_frames < 1 || tokens_per_frame < 1 || first_query_frame < 0 ||
        num_anchor < 0 || window < 1 || summary_tokens < 0 || summary_tokens > tokens_per_frame ||
        softmax_scale < 0.f)
        return GCA_ERR_INVALID_ARG;
    if (page_size != 64 && page_size != 128) return GCA_ERR_UNSUPPORTED;
    if (!is_device_ptr(k_pool) || !is_device_ptr(v_pool) || !is_device_ptr(q) || !is_device_ptr(out) ||
        (lse && !is_device_ptr(lse)) || (status && !is_device_ptr(status)))
        return GCA_ERR_INVALID_ARG;
    // the kernel moves 16-byte vectors through the pools (TMA), q and out,
    // and 4-byte words through lse, status and a device walk list
    auto off = [](const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) != 0; };
    if (off(k_pool, 16) || off(v_pool, 16) || off(q, 16) || off(out, 16) || off(lse, 4) || off(status, 4) ||
        off(walk, 4))
        return GCA_ERR_INVALID_ARG;
    if (nwalk > kNoallocMaxWalk) return GCA_ERR_CAPACITY;
    const long long R = (long long)num_query_frames * tokens_per_frame;
    const int QT = (int)((R + 127) / 128);
    // partial tiles used: at most QT * (W + H - 1); shrink the worker count to fit
    if ((long long)QT * num_heads > kNoallocMaxSlots) return GCA_ERR_CAPACITY;

    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess) return GCA_ERR_CUDA;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    unsigned char* base = scratch_address(dev);
    if (!base) return GCA_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    // every buffer the kernels touch must hold what the sizes say
    const size_t pool_bytes = (size_t)num_layers * num_pages * num_heads * page_size * gca::kHeadDim * 2;
    const size_t qo_bytes = (size_t)R * num_heads * gca::kHeadDim * 2;
    if (!fits_allocation(k_pool, pool_bytes) || !fits_allocation(v_pool, pool_bytes) ||
        !fits_allocation(q, qo_bytes) || !fits_allocation(out, qo_bytes) ||
        (lse && !fits_allocation(lse, (size_t)R * num_heads * sizeof(float))) ||
        (status && !fits_allocation(status, sizeof(int32_t))))
        return GCA_ERR_INVALID_ARG;
    const bool walk_on_host = !is_device_ptr(walk);
    if (walk_on_host) {
        // a host walk list is checked here; a device one by the kernel (status word)
        for (int i = 0; i < nwalk; ++i) {
            const gca_page_entry_t& e = walk[i];
            if (e.page_id < 0 || e.page_id >= num_pages || e.n_valid < 0 || e.n_valid > page_size ||
                (e.kind != GCA_PAGE_IMAGE && e.kind != GCA_PAGE_SUMMARY))
                return GCA_ERR_INVALID_ARG;
        }
    } else if (!fits_allocation(walk, sizeof(gca_page_entry_t) * (size_t)nwalk)) {
        return GCA_ERR_INVALID_ARG;
    }
    int* d_status = reinterpret_cast<int*>(base);
    unsigned long long* counts = reinterpret_cast<unsigned long long*>(base + kStatusBytes);
    unsigned char* rest = base + kStatusBytes + kCountBytes;
    gca_page_entry_t* walk_raw = reinterpret_cast<gca_page_entry_t*>(rest);
    int4* walk_dev = reinterpret_cast<int4*>(rest + kWalkRawBytes);
    float* ws_lse = reinterpret_cast<float*>(rest + kWalkRawBytes + kWalkBytes);
    float* ws_o = reinterpret_cast<float*>(rest + kWalkRawBytes + kWalkBytes + kLseBytes);

    const gca_page_entry_t* src = walk;
    if (walk_on_host) {
        if (cudaMemcpyAsync(walk_raw, walk, sizeof(gca_page_entry_t) * nwalk, cudaMemcpyHostToDevice, st) != cudaSuccess)
            return GCA_ERR_CUDA;
        src = walk_raw;
    }
    walk_to_int4<<<(nwalk + 255) / 256, 256, 0, st>>>(src, walk_dev, nwalk);
    if (cudaGetLastError() != cudaSuccess) return GCA_ERR_CUDA;

    CUtensorMap tk, tv;
    const cuuint64_t rows = (cuuint64_t)num_layers * num_pages * num_heads * page_size;
    cuuint64_t dims[2] = {(cuuint64_t)gca::kHeadDim, rows};
    cuuint64_t strides[1] = {(cuuint64_t)gca::kHeadDim * 2};
    cuuint32_t box[2] = {(cuuint32_t)gca::kHeadDim, (cuuint32_t)page_size};
    cuuint32_t estr[2] = {1, 1};
    for (int i = 0; i < 2; ++i) {
        if (g_encode(i ? &tv : &tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(i ? v_pool : k_pool),
                     dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return GCA_ERR_INVALID_ARG;
    }

    gca::AttendParams p{};
    p.walk = walk_dev;
    p.nwalk = nwalk;
    p.q = q;
    p.out = out;
    p.lse = lse;
    p.R = (int)R;
    p.H = num_heads;
    p.Lq = tokens_per_frame;
    p.first_query_frame = first_query_frame;
    p.rule = {num_anchor, window, summary_tokens, anchor_block ? 1 : 0};
    p.scale = softmax_scale > 0.f ? softmax_scale : 0.125f;   // 1/sqrt(64)
    p.scale_log2 = p.scale * 1.4426950408889634f;
    p.layer = layer;
    p.num_pages = num_pages;
    p.P = page_size;
    p.status = status ? status : d_status;
    p.ws_o = ws_o;
    p.ws_lse = ws_lse;
    p.QT = QT;
    // keep QT * (W + H - 1) partial tiles inside the scratch array
    gca::split_work(sms, (QT + 1) / 2, num_heads, nwalk, (long long)kNoallocMaxSlots / QT - num_heads + 1, &p.W,
                    &p.seg);
    p.merge_cnt = counts;
    p.epoch = g_epoch.fetch_add(1) + 1;
    p.frame_page0 = INT_MAX;
    cudaError_t err = gca::launch_attend_sm100(tk, tv, tk, tv, p, st);
    if (err != cudaSuccess) {
        cudaGetLastError();
        return GCA_ERR_CUDA;
    }
    return GCA_OK;
}
