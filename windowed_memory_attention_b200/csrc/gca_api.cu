// C ABI of the GCA hot path: the host page table and the launches.
//
// Host state per cache: one page table shared by every layer (the page ids of
// a frame are the same in all L pools), the frame counter, and for each layer
// the number of frames it has appended.  Device state: the two pools
// [L][num_pages][H][P][D], their TMA descriptors, the walk list, the split-KV
// scratch and the host-mapped status word.
//
// Page-table rules (the pages fix only that the cache is paged and sized for
// scale frames + window + slack; code walkthrough §3.4):
//   * pages are taken smallest free id first, in token order within a frame:
//     a new summary page when the frame's summary tokens reach one, then the
//     frame's ceil(M/P) image pages;
//   * the first `keep` special tokens of a frame form its trajectory memory
//     (keep = S by default; 1 keeps only the camera token; 0 keeps nothing):
//     token s < keep of frame t sits at stream index keep*t+s, page
//     (keep*t+s)/P of the summary stream, slot (keep*t+s)%P; the frame's other
//     S-keep special tokens and its M image tokens fill its image pages, in
//     token order (slot tau-keep), and leave with them at eviction;
//   * eviction after frame t returns the image pages of every non-anchor frame
//     f <= t-k (code walkthrough §2) — no bytes move;
//   * the walk list is the image pages of the full frames some query frame of
//     the block may see (ascending frame, then page), then every summary page;
//   * ceil((S+M)/P) transient pages sit after the allocator's pages: a
//     non-keyframe's K and V go there for one attention and are never kept.
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <map>
#include <set>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "../../include/gca.h"
#include "gca_internal.h"

using gca::WalkEntry;

namespace {

constexpr int kRing = 4;       // pinned staging slots for walk-list uploads
constexpr int kQRing = 8;      // device staging slots for host query blocks
constexpr int kORing = 2;      // device staging slots for host output blocks
constexpr int kMaxBatch = 64;  // frames per launch of batched frame attention
constexpr int kTileRows = 128;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

int ceil_div(long long a, long long b) { return (int)((a + b - 1) / b); }

}  // namespace

struct gca_cache {
    gca_config_t cfg{};
    int device = 0;
    int sms = 148;
    int P = 128, ipf = 1, num_pages = 0, Lq = 0;
    int keep = 0;          // special tokens per frame kept in the summary stream
    int ftok = 0;          // tokens in a full frame's image pages: Lq - keep
    int num_regular = 0;   // pages the allocator hands out; the transient pages follow
    int tpf = 0;           // transient pages: ceil(Lq / P)
    size_t elem = 2;
    float scale = 0.f;

    // page table
    std::set<int> free_pages;
    std::map<int, std::vector<int>> image_pages;   // full frames
    std::vector<int> summary_pages;
    std::vector<int> summary_opened_by;            // frame that opened each summary page
    int T = 0;
    std::vector<int> layer_frames;
    unsigned long long version = 1;

    // device memory
    void* kpool = nullptr;
    void* vpool = nullptr;
    size_t pool_bytes = 0;
    CUtensorMap tmK{}, tmV{};
    EncodeTiledFn encode = nullptr;   // cuTensorMapEncodeTiled (driver entry point)
    WalkEntry* d_walk = nullptr;
    int walk_cap = 0;
    WalkEntry* h_stage[kRing] = {};
    cudaEvent_t stage_ev[kRing] = {};
    int ring_pos = 0;
    unsigned long long up_version = 0;
    int up_F = -1;
    int up_n = 0;
    WalkEntry* d_walk_t = nullptr;   // walk list of the transient (non-keyframe) attention
    WalkEntry* d_walk_f = nullptr;   // the transient pages alone (frame attention)
    WalkEntry* d_walk_b = nullptr;   // kMaxBatch frames' own pages (batched frame attention)
    unsigned long long tup_version = 0;
    int tup_n = 0;
    float* ws_o = nullptr;
    float* ws_lse = nullptr;
    unsigned long long* merge_cnt = nullptr;   // [QT_max][H] split-head counters
    unsigned int epoch = 0;                    // launches of the bf16 kernel
    size_t ws_slots = 0;
    int* h_status = nullptr;
    int* d_status = nullptr;
    // staging for host-memory arguments: inputs are copied on the library's own
    // copy streams (so uploads overlap the kernels), guarded by events; outputs
    // are written to device staging and copied back on copy_out
    cudaStream_t copy = nullptr;      // query-block uploads (ring of staging slots)
    cudaStream_t copy_kv = nullptr;   // K/V uploads, so they never queue behind the ring
    cudaStream_t copy_out = nullptr;  // output blocks back to host memory
    void* st_k = nullptr;
    void* st_v = nullptr;
    cudaEvent_t kv_free = nullptr, kv_ready = nullptr;
    void* st_q[kQRing] = {};
    cudaEvent_t q_free[kQRing] = {}, q_ready[kQRing] = {};
    int q_pos = 0;
    void* st_out[kORing] = {};
    float* st_lse[kORing] = {};
    cudaEvent_t o_free[kORing] = {};
    cudaEvent_t o_ready = nullptr;
    int o_pos = 0;
    // device work of calls whose pointer arguments all live in host memory
    // (see begin_call); ev_fork / ev_join order it against the caller's stream
    cudaStream_t xs = nullptr;
    cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
    bool on_xs = false;               // the cache's latest device work is on xs
    long long launches = 0;
    bool host_only = false;   // GCA_HOST_ONLY: the page table alone, no device state
    // 3D rotary encoding: (cos, sin) tables of the time pairs per frame index
    // and of the spatial pairs per token of a frame
    float2* rope_t = nullptr;
    float2* rope_sp = nullptr;
    int rope_max_t = 0;
    gca::RopeTables rope() const { return {rope_t, rope_sp, rope_max_t}; }
};

namespace {

void release(gca_cache* c) {
    if (!c) return;
    if (c->host_only) {
        delete c->h_status;
        delete c;
        return;
    }
    int prev = 0;
    cudaGetDevice(&prev);
    cudaSetDevice(c->device);
    cudaFree(c->kpool);
    cudaFree(c->vpool);
    cudaFree(c->d_walk);
    cudaFree(c->d_walk_t);
    cudaFree(c->d_walk_f);
    cudaFree(c->d_walk_b);
    cudaFree(c->ws_o);
    cudaFree(c->ws_lse);
    cudaFree(c->merge_cnt);
    cudaFree(c->st_k);
    cudaFree(c->st_v);
    for (int i = 0; i < kQRing; ++i) {
        cudaFree(c->st_q[i]);
        if (c->q_free[i]) cudaEventDestroy(c->q_free[i]);
        if (c->q_ready[i]) cudaEventDestroy(c->q_ready[i]);
    }
    for (int i = 0; i < kORing; ++i) {
        cudaFree(c->st_out[i]);
        cudaFree(c->st_lse[i]);
        if (c->o_free[i]) cudaEventDestroy(c->o_free[i]);
    }
    if (c->o_ready) cudaEventDestroy(c->o_ready);
    if (c->ev_fork) cudaEventDestroy(c->ev_fork);
    if (c->ev_join) cudaEventDestroy(c->ev_join);
    if (c->copy_out) cudaStreamDestroy(c->copy_out);
    if (c->xs) cudaStreamDestroy(c->xs);
    cudaFree(c->rope_t);
    cudaFree(c->rope_sp);
    if (c->kv_free) cudaEventDestroy(c->kv_free);
    if (c->kv_ready) cudaEventDestroy(c->kv_ready);
    if (c->copy) cudaStreamDestroy(c->copy);
    if (c->copy_kv) cudaStreamDestroy(c->copy_kv);
    for (int i = 0; i < kRing; ++i) {
        if (c->h_stage[i]) cudaFreeHost(c->h_stage[i]);
        if (c->stage_ev[i]) cudaEventDestroy(c->stage_ev[i]);
    }
    if (c->h_status) cudaFreeHost(c->h_status);
    cudaSetDevice(prev);
    delete c;
}

// An NVTX range around one public call (a no-op unless a profiler attached one).
struct Range {
    explicit Range(const char* name) { nvtxRangePushA(name); }
    ~Range() { nvtxRangePop(); }
};

// Restores the caller's current device on scope exit.
struct DeviceGuard {
    int prev = -1;
    bool active = false;      // a host-only cache (device < 0) touches no device
    explicit DeviceGuard(int dev) : active(dev >= 0) {
        if (!active) return;
        cudaGetDevice(&prev);
        if (prev != dev) cudaSetDevice(dev);
    }
    ~DeviceGuard() {
        if (!active) return;
        int now = -1;
        cudaGetDevice(&now);
        if (prev >= 0 && now != prev) cudaSetDevice(prev);
    }
};

// Where a caller's pointer lives: device (or managed) memory is used in place;
// pinned and pageable host memory are staged through library buffers.
enum class Mem { kDevice, kPinned, kPageable };

Mem classify(const void* ptr) {
    cudaPointerAttributes a{};
    if (cudaPointerGetAttributes(&a, ptr) != cudaSuccess) {
        cudaGetLastError();
        return Mem::kPageable;
    }
    if (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) return Mem::kDevice;
    return a.type == cudaMemoryTypeHost ? Mem::kPinned : Mem::kPageable;
}

bool is_device_ptr(const void* ptr) { return classify(ptr) == Mem::kDevice; }

// The stream a call's device work runs on.  A call whose pointer arguments
// all live in host memory reads nothing that earlier work on the caller's
// stream writes: its inputs are staged and its outputs copied back by the
// library.  Its work runs on the cache's own stream xs, after the cache's
// earlier work only, so the copy back of one call overlaps the kernels of the
// next; end_call makes the caller's stream wait for the call.  Any other call
// runs on the caller's stream.
bool begin_call(gca_cache* c, cudaStream_t st, bool detached, cudaStream_t* ex) {
    *ex = st;
    if (!detached) {
        // the cache's work on xs, if any, is already waited for by st (end_call)
        c->on_xs = false;
        return true;
    }
    if (!c->on_xs && (cudaEventRecord(c->ev_fork, st) != cudaSuccess ||
                      cudaStreamWaitEvent(c->xs, c->ev_fork, 0) != cudaSuccess))
        return false;
    c->on_xs = true;
    *ex = c->xs;
    return true;
}

int end_call(gca_cache* c, cudaStream_t st, cudaStream_t ex, int rc) {
    if (ex != st && (cudaEventRecord(c->ev_join, ex) != cudaSuccess ||
                     cudaStreamWaitEvent(st, c->ev_join, 0) != cudaSuccess))
        return rc ? rc : GCA_ERR_CUDA;
    return rc;
}

bool on_host(const void* ptr) { return ptr && classify(ptr) != Mem::kDevice; }

// The kernels move 16-byte vectors through q, k, v and out and 4-byte words
// through lse: a device pointer must start on such a boundary (allocations
// do).  Host pointers may sit anywhere: they are staged through aligned
// library buffers.
bool placed(const void* ptr, uintptr_t align) {
    return !ptr || (reinterpret_cast<uintptr_t>(ptr) % align) == 0 || on_host(ptr);
}

// Upload a host query block into a staging slot on the cache's copy stream: the
// copy waits until the buffer's previous reader (on the caller's stream) is
// done (`free_ev`), and the caller's stream waits for the copy (`ready_ev`).
// The caller records free_ev on its stream after the kernel that reads dst.
bool stage_in(gca_cache* c, void* dst, const void* src, size_t bytes, cudaEvent_t free_ev,
              cudaEvent_t ready_ev, cudaStream_t st) {
    return cudaStreamWaitEvent(c->copy, free_ev, 0) == cudaSuccess &&
           cudaMemcpyAsync(dst, src, bytes, cudaMemcpyHostToDevice, c->copy) == cudaSuccess &&
           cudaEventRecord(ready_ev, c->copy) == cudaSuccess &&
           cudaStreamWaitEvent(st, ready_ev, 0) == cudaSuccess;
}

// K and V of a frame (or of all layers) from the caller, staged when on the host.
bool stage_kv(gca_cache* c, const void* k, const void* v, size_t bytes, cudaStream_t st,
              const void** kd, const void** vd) {
    *kd = k;
    *vd = v;
    const bool kh = !is_device_ptr(k), vh = !is_device_ptr(v);
    if (!kh && !vh) return true;
    if (cudaStreamWaitEvent(c->copy_kv, c->kv_free, 0) != cudaSuccess) return false;
    if (kh) {
        if (cudaMemcpyAsync(c->st_k, k, bytes, cudaMemcpyHostToDevice, c->copy_kv) != cudaSuccess) return false;
        *kd = c->st_k;
    }
    if (vh) {
        if (cudaMemcpyAsync(c->st_v, v, bytes, cudaMemcpyHostToDevice, c->copy_kv) != cudaSuccess) return false;
        *vd = c->st_v;
    }
    return cudaEventRecord(c->kv_ready, c->copy_kv) == cudaSuccess &&
           cudaStreamWaitEvent(st, c->kv_ready, 0) == cudaSuccess;
}

bool encode_pool_map(EncodeTiledFn enc, CUtensorMap* tm, void* pool, const gca_cache* c) {
    const cuuint64_t rows = (cuuint64_t)c->cfg.num_layers * c->num_pages * c->cfg.num_heads * c->P;
    cuuint64_t dims[2] = {(cuuint64_t)gca::kHeadDim, rows};
    cuuint64_t strides[1] = {(cuuint64_t)gca::kHeadDim * 2};
    cuuint32_t box[2] = {(cuuint32_t)gca::kHeadDim, (cuuint32_t)c->P};
    cuuint32_t estr[2] = {1, 1};
    return enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, pool, dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

// A frame's K or V as the caller passes it, [S+M][H][D] bf16, viewed as a 3D
// tensor (D, H, token): a box of D x 1 x P is one head's tile of P tokens,
// laid out in shared memory exactly like a pool page tile; boxes past the
// last token read zeros.
bool encode_frame_map(const gca_cache* c, CUtensorMap* tm, const void* base, int frames = 1) {
    if (!c->encode || (reinterpret_cast<uintptr_t>(base) & 15u)) return false;
    const cuuint64_t H = (cuuint64_t)c->cfg.num_heads;
    cuuint64_t dims[3] = {(cuuint64_t)gca::kHeadDim, H, (cuuint64_t)c->Lq * (cuuint64_t)frames};
    cuuint64_t strides[2] = {(cuuint64_t)gca::kHeadDim * 2, H * gca::kHeadDim * 2};
    cuuint32_t box[3] = {(cuuint32_t)gca::kHeadDim, 1, (cuuint32_t)c->P};
    cuuint32_t estr[3] = {1, 1, 1};
    return c->encode(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
                     estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Host tables of the 3D rotary encoding.  Axis a (time, patch row, patch
// column) owns d_a = 24, 20, 20 head dims; its pair i turns by
// pos * base^(-2i/d_a).  Angles are formed in double and stored as float.
bool build_rope_tables(gca_cache* c) {
    const gca_config_t& g = c->cfg;
    const double base = g.rope_base > 0.f ? (double)g.rope_base : 10000.0;
    const int gw = g.rope_grid_w > 0 ? g.rope_grid_w : g.image_tokens;
    auto freq = [&](int i, int d) { return std::pow(base, -2.0 * i / d); };
    c->rope_max_t = g.max_frames;
    std::vector<float2> ht((size_t)c->rope_max_t * gca::kRopeTPairs);
    for (int t = 0; t < c->rope_max_t; ++t)
        for (int i = 0; i < gca::kRopeTPairs; ++i) {
            const double a = t * freq(i, 2 * gca::kRopeTPairs);
            ht[(size_t)t * gca::kRopeTPairs + i] = make_float2((float)std::cos(a), (float)std::sin(a));
        }
    std::vector<float2> hs((size_t)c->Lq * gca::kRopeSpPairs);
    constexpr int kYPairs = gca::kRopeSpPairs / 2;         // 10 pairs each for row and column
    for (int u = 0; u < c->Lq; ++u) {
        const int m = u - g.summary_tokens;                 // image token index, < 0: special
        const int y = m < 0 ? 0 : m / gw, x = m < 0 ? 0 : m % gw;
        for (int i = 0; i < gca::kRopeSpPairs; ++i) {
            const int pos = i < kYPairs ? y : x;
            const double a = pos * freq(i % kYPairs, 2 * kYPairs);
            hs[(size_t)u * gca::kRopeSpPairs + i] = make_float2((float)std::cos(a), (float)std::sin(a));
        }
    }
    return cudaMalloc(&c->rope_t, ht.size() * sizeof(float2)) == cudaSuccess &&
           cudaMalloc(&c->rope_sp, hs.size() * sizeof(float2)) == cudaSuccess &&
           cudaMemcpy(c->rope_t, ht.data(), ht.size() * sizeof(float2), cudaMemcpyHostToDevice) == cudaSuccess &&
           cudaMemcpy(c->rope_sp, hs.data(), hs.size() * sizeof(float2), cudaMemcpyHostToDevice) == cudaSuccess;
}

bool frame_seen(const gca_cache* c, int i, int j) {
    const int n = c->cfg.num_anchor, k = c->cfg.window;
    if (c->cfg.anchor_block && i < n && j < n) return true;
    return j <= i && (j < n || j >= i - k + 1);
}

// walk list for the block of the F latest frames; false if a needed frame was evicted
bool build_walk(const gca_cache* c, int F, std::vector<gca_page_entry_t>& out) {
    out.clear();
    const int q0 = c->T - F;
    for (int i = q0; i < c->T; ++i)
        for (int j = 0; j < c->T; ++j)
            if (frame_seen(c, i, j) && !c->image_pages.count(j)) return false;
    for (const auto& kv : c->image_pages) {
        bool seen = false;
        for (int i = q0; i < c->T && !seen; ++i) seen = frame_seen(c, i, kv.first);
        if (!seen) continue;
        for (size_t s = 0; s < kv.second.size(); ++s) {
            const int first = (int)s * c->P;
            out.push_back({kv.second[s], GCA_PAGE_IMAGE, kv.first, first,
                           std::min(c->P, c->ftok - first)});
        }
    }
    const long long total = (long long)c->keep * c->T;
    for (size_t s = 0; s < c->summary_pages.size(); ++s) {
        const int first = (int)s * c->P;
        out.push_back({c->summary_pages[s], GCA_PAGE_SUMMARY, first / c->keep, first,
                       (int)std::min<long long>(c->P, total - first)});
    }
    return true;
}

// Stages a walk list through the pinned ring and copies it to dst on st.
int upload_walk(gca_cache* c, const std::vector<gca_page_entry_t>& w, WalkEntry* dst, cudaStream_t st) {
    if ((int)w.size() > c->walk_cap) return GCA_ERR_CAPACITY;
    const int slot = c->ring_pos;
    c->ring_pos = (c->ring_pos + 1) % kRing;
    if (cudaEventSynchronize(c->stage_ev[slot]) != cudaSuccess) return GCA_ERR_CUDA;
    WalkEntry* hs = c->h_stage[slot];
    for (size_t i = 0; i < w.size(); ++i) {
        const gca_page_entry_t& e = w[i];
        hs[i] = make_int4(e.page_id, e.n_valid, e.first, e.kind == GCA_PAGE_IMAGE ? e.frame : -1);
    }
    if (cudaMemcpyAsync(dst, hs, sizeof(WalkEntry) * w.size(), cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaEventRecord(c->stage_ev[slot], st) != cudaSuccess)
        return GCA_ERR_CUDA;
    return GCA_OK;
}

// Attention of F query frames (the first is first_query_frame) over a device
// walk list; stages host q / out / lse through the cache's buffers.
// fk / fv (nullable): the query frame's own K and V, read in place by the
// kernel for the transient pages (ids >= num_regular) of the walk list.
int run_attention(gca_cache* c, int layer, const void* q, int F, int first_query_frame,
                  const WalkEntry* walk, int nwalk, void* out, float* lse, cudaStream_t ex,
                  cudaStream_t st, const CUtensorMap* fk = nullptr, const CUtensorMap* fv = nullptr) {
    const gca_config_t& g = c->cfg;
    const int R = F * c->Lq;
    const size_t qbytes = (size_t)R * g.num_heads * gca::kHeadDim * c->elem;
    const void* qd = q;
    int qslot = -1;
    if (!is_device_ptr(q)) {
        qslot = c->q_pos;
        c->q_pos = (c->q_pos + 1) % kQRing;
        if (!stage_in(c, c->st_q[qslot], q, qbytes, c->q_free[qslot], c->q_ready[qslot], ex))
            return GCA_ERR_CUDA;
        qd = c->st_q[qslot];
    }
    // outputs in host memory (pinned or pageable) are written to a device
    // staging slot by the kernel and copied back by the copy engine, which
    // moves them at PCIe rate; kernel stores into a mapped pinned buffer
    // stall the CTAs that issue them
    const bool out_host = on_host(out);
    const bool lse_host = on_host(lse);
    int oslot = -1;
    if (out_host || lse_host) {
        oslot = c->o_pos;
        c->o_pos = (c->o_pos + 1) % kORing;
        // the slot's previous copy back has read it
        if (cudaStreamWaitEvent(ex, c->o_free[oslot], 0) != cudaSuccess) return GCA_ERR_CUDA;
    }

    gca::AttendParams p{};
    p.walk = walk;
    p.nwalk = nwalk;
    p.q = qd;
    p.out = out_host ? c->st_out[oslot] : out;
    p.lse = lse ? (lse_host ? c->st_lse[oslot] : lse) : nullptr;
    p.R = R;
    p.H = g.num_heads;
    p.Lq = c->Lq;
    p.first_query_frame = first_query_frame;
    p.rule = {g.num_anchor, g.window, c->keep, g.anchor_block ? 1 : 0};
    p.scale = c->scale;
    p.scale_log2 = c->scale * 1.4426950408889634f;
    p.layer = layer;
    p.num_pages = c->num_pages;
    p.P = c->P;
    p.status = c->d_status;
    p.ws_o = c->ws_o;
    p.ws_lse = c->ws_lse;
    p.rope = c->rope();

    cudaError_t err;
    if (g.dtype == GCA_DTYPE_BF16) {
        // split: QT query tiles x W workers over the head-major page stream
        p.QT = ceil_div(R, kTileRows);
        gca::split_work(c->sms, (p.QT + 1) / 2, g.num_heads, p.nwalk, LLONG_MAX, &p.W, &p.seg);
        p.merge_cnt = c->merge_cnt;
        p.epoch = ++c->epoch;
        p.frame_page0 = fk && fv ? c->num_regular : INT_MAX;
        err = gca::launch_attend_sm100(c->tmK, c->tmV, fk ? *fk : c->tmK, fv ? *fv : c->tmV, p, ex);
        c->launches += 1;
    } else {
        p.QT = ceil_div(R, kTileRows);
        p.W = 1;
        p.seg = 1;
        err = gca::launch_attend_f32(p, c->kpool, c->vpool, ex);
        c->launches += 1;
    }
    if (err != cudaSuccess) {
        cudaGetLastError();
        return GCA_ERR_CUDA;
    }
    if (qslot >= 0 && cudaEventRecord(c->q_free[qslot], ex) != cudaSuccess) return GCA_ERR_CUDA;
    if (oslot >= 0) {
        // copy back on copy_out when the call runs on xs (the next call's
        // kernels go on while it runs), else in the caller's stream order
        cudaStream_t cs = ex == st ? st : c->copy_out;
        if (cs != ex && (cudaEventRecord(c->o_ready, ex) != cudaSuccess ||
                         cudaStreamWaitEvent(cs, c->o_ready, 0) != cudaSuccess))
            return GCA_ERR_CUDA;
        if (out_host && cudaMemcpyAsync(out, c->st_out[oslot], qbytes, cudaMemcpyDeviceToHost, cs) != cudaSuccess)
            return GCA_ERR_CUDA;
        if (lse_host && cudaMemcpyAsync(lse, c->st_lse[oslot], (size_t)R * g.num_heads * sizeof(float),
                                        cudaMemcpyDeviceToHost, cs) != cudaSuccess)
            return GCA_ERR_CUDA;
        if (cudaEventRecord(c->o_free[oslot], cs) != cudaSuccess) return GCA_ERR_CUDA;
        if (cs != st && cudaStreamWaitEvent(st, c->o_free[oslot], 0) != cudaSuccess) return GCA_ERR_CUDA;
    }
    return GCA_OK;
}

// A frame's K and V for attention over its own tokens.  bf16 without RoPE:
// the attention kernel reads them in place through *fk / *fv (host inputs
// are staged first) and *direct is set; the caller records kv_free after the
// attention kernel.  Otherwise append_kernel writes them into this layer's
// transient pages: token u of the frame (summary tokens first) at page u / P,
// slot u % P.
int stage_transient(gca_cache* c, int layer, const void* k, const void* v, int frame, cudaStream_t st,
                    CUtensorMap* fk, CUtensorMap* fv, bool* direct) {
    const gca_config_t& g = c->cfg;
    gca::AppendParams p{};
    const size_t bytes = (size_t)c->Lq * g.num_heads * gca::kHeadDim * c->elem;
    if (!stage_kv(c, k, v, bytes, st, &p.k, &p.v)) return GCA_ERR_CUDA;
    *direct = g.dtype == GCA_DTYPE_BF16 && g.rope == GCA_ROPE_NONE && encode_frame_map(c, fk, p.k) &&
              encode_frame_map(c, fv, p.v);
    if (*direct) return GCA_OK;
    p.kpool = c->kpool;
    p.vpool = c->vpool;
    p.layer0 = layer;
    p.nlayers = 1;
    p.Lq = c->Lq;
    p.S = 0;                 // every token of the frame is laid out like an image token
    p.M = c->Lq;
    p.H = g.num_heads;
    p.P = c->P;
    p.num_pages = c->num_pages;
    p.elem_bytes = (int)c->elem;
    p.sms = c->sms;
    p.frame = frame;
    p.sum_seq0 = 0;
    p.sum_page[0] = p.sum_page[1] = -1;
    p.new_sum_seq = -1;
    for (int s = 0; s < c->tpf; ++s) p.img_pages[s] = c->num_regular + s;
    p.rope = c->rope();
    p.rope_t = frame;
    if (gca::launch_append(p, st) != cudaSuccess) {
        cudaGetLastError();
        return GCA_ERR_CUDA;
    }
    c->launches += 1;
    if (cudaEventRecord(c->kv_free, st) != cudaSuccess) return GCA_ERR_CUDA;
    return GCA_OK;
}

int check_status(const gca_cache* c) {
    return (*(volatile int*)c->h_status) ? GCA_ERR_DEVICE_CHECK : GCA_OK;
}

}  // namespace

extern "C" {

const char* gca_status_string(int s) {
    switch (s) {
        case GCA_OK: return "ok";
        case GCA_ERR_INVALID_ARG: return "invalid argument";
        case GCA_ERR_CAPACITY: return "capacity exhausted";
        case GCA_ERR_STATE: return "call out of order";
        case GCA_ERR_UNSUPPORTED: return "unsupported configuration";
        case GCA_ERR_CUDA: return "CUDA error";
        case GCA_ERR_DEVICE_CHECK: return "device status word raised";
        default: return "unknown status";
    }
}

int gca_cache_create(const gca_config_t* cfg, int device, gca_cache_t** out) {
    if (!cfg || !out) return GCA_ERR_INVALID_ARG;
    *out = nullptr;
    const gca_config_t& g = *cfg;
    if (g.num_layers < 1 || g.num_heads < 1 || g.image_tokens < 1 || g.summary_tokens < 1 ||
        g.num_anchor < 0 || g.window < 1 || g.max_frames < 1 || g.max_query_frames < 1 ||
        g.frame_slack < 0 || g.softmax_scale < 0.f || g.trajectory_memory < GCA_MEMORY_SUMMARY ||
        g.trajectory_memory > GCA_MEMORY_NONE || g.rope < GCA_ROPE_NONE || g.rope > GCA_ROPE_3D ||
        g.rope_grid_w < 0 || g.rope_base < 0.f)
        return GCA_ERR_INVALID_ARG;
    if (g.head_dim != gca::kHeadDim || (g.page_size != 64 && g.page_size != 128) ||
        (g.dtype != GCA_DTYPE_BF16 && g.dtype != GCA_DTYPE_F32))
        return GCA_ERR_UNSUPPORTED;
    // a frame's image pages, and a non-keyframe's transient pages, fit one append launch
    if ((g.image_tokens + g.summary_tokens + g.page_size - 1) / g.page_size > gca::kMaxImagePages)
        return GCA_ERR_UNSUPPORTED;
    const bool host = device == GCA_HOST_ONLY;
    int ndev = 0;
    if (!host && (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev)) {
        cudaGetLastError();
        return GCA_ERR_INVALID_ARG;
    }
    DeviceGuard guard(device);

    gca_cache* c = new gca_cache();
    c->cfg = g;
    c->device = device;
    c->host_only = host;
    if (!host) cudaDeviceGetAttribute(&c->sms, cudaDevAttrMultiProcessorCount, device);
    c->P = g.page_size;
    c->keep = g.trajectory_memory == GCA_MEMORY_SUMMARY ? g.summary_tokens
            : g.trajectory_memory == GCA_MEMORY_CAMERA ? 1 : 0;
    c->ftok = g.image_tokens + g.summary_tokens - c->keep;
    c->ipf = ceil_div(c->ftok, c->P);
    const long long image_cap = (long long)(g.num_anchor + g.window + g.max_query_frames + g.frame_slack) * c->ipf;
    const long long summary_cap = ceil_div((long long)c->keep * g.max_frames, c->P);
    if (image_cap + summary_cap > (1LL << 30)) { delete c; return GCA_ERR_CAPACITY; }
    c->Lq = g.image_tokens + g.summary_tokens;
    c->num_regular = (int)(image_cap + summary_cap);
    c->tpf = ceil_div(c->Lq, c->P);
    c->num_pages = c->num_regular + c->tpf;
    c->elem = g.dtype == GCA_DTYPE_BF16 ? 2 : 4;
    c->scale = g.softmax_scale > 0.f ? g.softmax_scale : 1.0f / sqrtf((float)g.head_dim);
    c->layer_frames.assign(g.num_layers, 0);
    for (int i = 0; i < c->num_regular; ++i) c->free_pages.insert(i);

    const size_t tile = (size_t)c->P * gca::kHeadDim * c->elem;
    c->pool_bytes = (size_t)g.num_layers * c->num_pages * g.num_heads * tile;
    c->walk_cap = c->num_pages;
    if (host) {
        c->h_status = new int(0);
        *out = c;
        return GCA_OK;
    }
    bool ok = cudaMalloc(&c->kpool, c->pool_bytes) == cudaSuccess &&
              cudaMalloc(&c->vpool, c->pool_bytes) == cudaSuccess;
    ok = ok && cudaMalloc(&c->d_walk, sizeof(WalkEntry) * c->walk_cap) == cudaSuccess &&
         cudaMalloc(&c->d_walk_t, sizeof(WalkEntry) * c->walk_cap) == cudaSuccess &&
         cudaMalloc(&c->d_walk_f, sizeof(WalkEntry) * c->tpf) == cudaSuccess &&
         cudaMalloc(&c->d_walk_b, sizeof(WalkEntry) * c->tpf * kMaxBatch) == cudaSuccess;
    if (ok) {
        // frame attention reads the transient pages only, as frame 0; the
        // batched form gives frame f of a launch its own pages, whose tokens
        // start at f * (S+M) of the caller's [F][S+M][H][D] tensors
        std::vector<WalkEntry> wf(c->tpf), wb((size_t)c->tpf * kMaxBatch);
        for (int s = 0; s < c->tpf; ++s)
            wf[s] = make_int4(c->num_regular + s, std::min(c->P, c->Lq - s * c->P), s * c->P, 0);
        for (int f = 0; f < kMaxBatch; ++f)
            for (int s = 0; s < c->tpf; ++s)
                wb[(size_t)f * c->tpf + s] = make_int4(c->num_regular + s, std::min(c->P, c->Lq - s * c->P),
                                                       f * c->Lq + s * c->P, f);
        ok = cudaMemcpy(c->d_walk_f, wf.data(), sizeof(WalkEntry) * c->tpf, cudaMemcpyHostToDevice) ==
                 cudaSuccess &&
             cudaMemcpy(c->d_walk_b, wb.data(), sizeof(WalkEntry) * wb.size(), cudaMemcpyHostToDevice) ==
                 cudaSuccess;
    }
    for (int i = 0; ok && i < kRing; ++i) {
        ok = cudaHostAlloc((void**)&c->h_stage[i], sizeof(WalkEntry) * c->walk_cap, cudaHostAllocDefault) == cudaSuccess &&
             cudaEventCreateWithFlags(&c->stage_ev[i], cudaEventDisableTiming) == cudaSuccess;
    }
    // split-KV scratch: per 128-row query tile at most W + H - 1 (worker, head)
    // partials; W <= max(1, SMs / tile pairs), so QT * W <= 2 * max(SMs, pairs)
    const int qt_max = ceil_div((long long)g.max_query_frames * c->Lq, kTileRows);
    const int qp_max = (qt_max + 1) / 2;
    c->ws_slots = 2 * (size_t)std::max(c->sms, qp_max) + (size_t)qt_max * (g.num_heads - 1);
    if (g.dtype == GCA_DTYPE_BF16) {
        const size_t cnt_bytes = (size_t)qt_max * g.num_heads * sizeof(unsigned long long);
        ok = ok && cudaMalloc(&c->ws_o, c->ws_slots * kTileRows * gca::kHeadDim * sizeof(float)) == cudaSuccess &&
             cudaMalloc(&c->ws_lse, c->ws_slots * kTileRows * sizeof(float)) == cudaSuccess &&
             cudaMalloc(&c->merge_cnt, cnt_bytes) == cudaSuccess &&
             cudaMemset(c->merge_cnt, 0, cnt_bytes) == cudaSuccess;
    }
    ok = ok && cudaHostAlloc((void**)&c->h_status, sizeof(int), cudaHostAllocMapped) == cudaSuccess;
    if (ok) {
        *c->h_status = 0;
        ok = cudaHostGetDevicePointer((void**)&c->d_status, c->h_status, 0) == cudaSuccess;
    }
    const size_t frame_bytes = (size_t)c->Lq * g.num_heads * gca::kHeadDim * c->elem;
    ok = ok && cudaStreamCreateWithFlags(&c->copy, cudaStreamNonBlocking) == cudaSuccess &&
         cudaStreamCreateWithFlags(&c->copy_kv, cudaStreamNonBlocking) == cudaSuccess &&
         cudaEventCreateWithFlags(&c->kv_free, cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&c->kv_ready, cudaEventDisableTiming) == cudaSuccess;
    for (int i = 0; ok && i < kQRing; ++i)
        ok = cudaMalloc(&c->st_q[i], frame_bytes * g.max_query_frames) == cudaSuccess &&
             cudaEventCreateWithFlags(&c->q_free[i], cudaEventDisableTiming) == cudaSuccess &&
             cudaEventCreateWithFlags(&c->q_ready[i], cudaEventDisableTiming) == cudaSuccess;
    ok = ok && cudaMalloc(&c->st_k, frame_bytes * g.num_layers) == cudaSuccess &&
         cudaMalloc(&c->st_v, frame_bytes * g.num_layers) == cudaSuccess;
    for (int i = 0; ok && i < kORing; ++i)
        ok = cudaMalloc(&c->st_out[i], frame_bytes * g.max_query_frames) == cudaSuccess &&
             cudaMalloc((void**)&c->st_lse[i], (size_t)c->Lq * g.num_heads * g.max_query_frames * sizeof(float)) ==
                 cudaSuccess &&
             cudaEventCreateWithFlags(&c->o_free[i], cudaEventDisableTiming) == cudaSuccess;
    ok = ok && cudaStreamCreateWithFlags(&c->copy_out, cudaStreamNonBlocking) == cudaSuccess &&
         cudaStreamCreateWithFlags(&c->xs, cudaStreamNonBlocking) == cudaSuccess &&
         cudaEventCreateWithFlags(&c->o_ready, cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&c->ev_fork, cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&c->ev_join, cudaEventDisableTiming) == cudaSuccess;
    if (!ok) {
        cudaGetLastError();
        release(c);
        return GCA_ERR_CUDA;
    }
    if (g.rope == GCA_ROPE_3D && !build_rope_tables(c)) {
        cudaGetLastError();
        release(c);
        return GCA_ERR_CUDA;
    }
    if (g.dtype == GCA_DTYPE_BF16) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            !fn || !encode_pool_map((EncodeTiledFn)fn, &c->tmK, c->kpool, c) ||
            !encode_pool_map((EncodeTiledFn)fn, &c->tmV, c->vpool, c)) {
            cudaGetLastError();
            release(c);
            return GCA_ERR_CUDA;
        }
        c->encode = (EncodeTiledFn)fn;
    }
    *out = c;
    return GCA_OK;
}

int gca_cache_destroy(gca_cache_t* c) {
    release(c);
    return GCA_OK;
}

int gca_append_frame(gca_cache_t* c, int32_t layer, const void* k, const void* v,
                     int64_t* frame_index_out, void* stream) {
    Range range("gca_append_frame");
    if (!c || (!c->host_only && (!k || !v))) return GCA_ERR_INVALID_ARG;
    if (!c->host_only && (!placed(k, 16) || !placed(v, 16))) return GCA_ERR_INVALID_ARG;
    const gca_config_t& g = c->cfg;
    if (layer != GCA_ALL_LAYERS && (layer < 0 || layer >= g.num_layers)) return GCA_ERR_INVALID_ARG;
    if (int s = check_status(c)) return s;
    DeviceGuard guard(c->device);
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    int t, l0, nl;
    if (layer == GCA_ALL_LAYERS || layer == 0) {
        for (int l = 0; l < g.num_layers; ++l)
            if (c->layer_frames[l] != c->T) return GCA_ERR_STATE;
        if (c->T >= g.max_frames) return GCA_ERR_CAPACITY;
        t = c->T;
        const int S = c->keep;
        int new_sum = 0;
        for (int s = 0; s < S; ++s) new_sum += ((S * t + s) % c->P) == 0;
        if ((int)c->free_pages.size() < c->ipf + new_sum) return GCA_ERR_CAPACITY;
        auto take = [&]() {
            const int pid = *c->free_pages.begin();
            c->free_pages.erase(c->free_pages.begin());
            return pid;
        };
        for (int s = 0; s < S; ++s)
            if (((S * t + s) % c->P) == 0) {
                c->summary_pages.push_back(take());
                c->summary_opened_by.push_back(t);
            }
        std::vector<int> pages(c->ipf);
        for (int i = 0; i < c->ipf; ++i) pages[i] = take();
        c->image_pages[t] = pages;
        c->T += 1;
        c->version += 1;
        l0 = 0;
        nl = layer == GCA_ALL_LAYERS ? g.num_layers : 1;
    } else {
        if (c->T == 0 || c->layer_frames[layer] != c->T - 1) return GCA_ERR_STATE;
        t = c->T - 1;
        l0 = layer;
        nl = 1;
    }
    if (c->host_only) {       // page table only: nothing to copy
        for (int l = l0; l < l0 + nl; ++l) c->layer_frames[l] = t + 1;
        if (frame_index_out) *frame_index_out = t;
        return GCA_OK;
    }

    cudaStream_t ex;
    if (!begin_call(c, st, on_host(k) && on_host(v), &ex)) return GCA_ERR_CUDA;
    gca::AppendParams p{};
    const size_t bytes = (size_t)nl * c->Lq * g.num_heads * gca::kHeadDim * c->elem;
    if (!stage_kv(c, k, v, bytes, ex, &p.k, &p.v)) return end_call(c, st, ex, GCA_ERR_CUDA);
    p.kpool = c->kpool;
    p.vpool = c->vpool;
    p.layer0 = l0;
    p.nlayers = nl;
    p.Lq = c->Lq;
    p.S = c->keep;           // tokens s < keep go to the summary stream,
    p.M = c->ftok;           // the rest to the frame's image pages
    p.H = g.num_heads;
    p.P = c->P;
    p.num_pages = c->num_pages;
    p.elem_bytes = (int)c->elem;
    p.sms = c->sms;
    p.frame = t;
    const int S = c->keep;
    p.sum_seq0 = (S * t) / c->P;
    p.sum_page[0] = p.sum_seq0 < (int)c->summary_pages.size() ? c->summary_pages[p.sum_seq0] : -1;
    p.sum_page[1] = (p.sum_seq0 + 1 < (int)c->summary_pages.size()) ? c->summary_pages[p.sum_seq0 + 1] : -1;
    p.new_sum_seq = -1;
    for (int s = 0; s < S; ++s)
        if (((S * t + s) % c->P) == 0) p.new_sum_seq = (S * t + s) / c->P;
    const std::vector<int>& img = c->image_pages.at(t);
    for (int i = 0; i < c->ipf; ++i) p.img_pages[i] = img[i];
    p.rope = c->rope();
    p.rope_t = t;
    if (gca::launch_append(p, ex) != cudaSuccess) {
        cudaGetLastError();
        return end_call(c, st, ex, GCA_ERR_CUDA);
    }
    c->launches += 1;
    if (cudaEventRecord(c->kv_free, ex) != cudaSuccess) return end_call(c, st, ex, GCA_ERR_CUDA);
    for (int l = l0; l < l0 + nl; ++l) c->layer_frames[l] = t + 1;
    if (frame_index_out) *frame_index_out = t;
    return end_call(c, st, ex, GCA_OK);
}

int gca_evict_to_summary(gca_cache_t* c, int32_t* frames_evicted_out) {
    Range range("gca_evict_to_summary");
    if (!c) return GCA_ERR_INVALID_ARG;
    const int t = c->T - 1;
    int count = 0;
    for (auto it = c->image_pages.begin(); it != c->image_pages.end();) {
        const int f = it->first;
        if (f >= c->cfg.num_anchor && f <= t - c->cfg.window) {
            for (int pid : it->second) c->free_pages.insert(pid);
            it = c->image_pages.erase(it);
            ++count;
        } else {
            ++it;
        }
    }
    if (count) c->version += 1;
    if (frames_evicted_out) *frames_evicted_out = count;
    return GCA_OK;
}

int gca_reset(gca_cache_t* c) {
    Range range("gca_reset");
    if (!c) return GCA_ERR_INVALID_ARG;
    c->free_pages.clear();
    for (int i = 0; i < c->num_regular; ++i) c->free_pages.insert(i);
    c->image_pages.clear();
    c->summary_pages.clear();
    c->summary_opened_by.clear();
    c->T = 0;
    std::fill(c->layer_frames.begin(), c->layer_frames.end(), 0);
    c->version += 1;
    return GCA_OK;
}

int gca_get_layout(const gca_cache_t* c, int32_t F, gca_page_entry_t* out, int32_t cap, int32_t* n_out) {
    if (!c || !n_out || cap < 0 || (cap > 0 && !out)) return GCA_ERR_INVALID_ARG;
    if (F < 1 || F > c->T) return GCA_ERR_STATE;
    std::vector<gca_page_entry_t> w;
    if (!build_walk(c, F, w)) return GCA_ERR_STATE;
    const int n = (int)w.size();
    for (int i = 0; i < std::min(n, cap); ++i) out[i] = w[i];
    *n_out = n;
    return GCA_OK;
}

int gca_token_slot(const gca_cache_t* c, int32_t frame, int32_t tau, int32_t* page_id_out, int32_t* slot_out) {
    if (!c || !page_id_out || !slot_out) return GCA_ERR_INVALID_ARG;
    const int S = c->keep;
    if (frame < 0 || frame >= c->T || tau < 0 || tau >= c->Lq) return GCA_ERR_INVALID_ARG;
    if (tau < S) {
        const long long idx = (long long)S * frame + tau;
        *page_id_out = c->summary_pages[idx / c->P];
        *slot_out = (int)(idx % c->P);
        return GCA_OK;
    }
    auto it = c->image_pages.find(frame);
    if (it == c->image_pages.end()) return GCA_ERR_STATE;
    const int m = tau - S;
    *page_id_out = it->second[m / c->P];
    *slot_out = m % c->P;
    return GCA_OK;
}

int gca_visible_prefix(const gca_cache_t* c, const gca_page_entry_t* e, int32_t query_frame,
                       int32_t* prefix_out) {
    if (!c || !e || !prefix_out || query_frame < 0) return GCA_ERR_INVALID_ARG;
    const gca::MaskRule rule{c->cfg.num_anchor, c->cfg.window, c->keep, c->cfg.anchor_block ? 1 : 0};
    const int4 w = make_int4(e->page_id, e->n_valid, e->first, e->kind == GCA_PAGE_IMAGE ? e->frame : -1);
    *prefix_out = gca::visible_prefix(rule, w, query_frame);
    return GCA_OK;
}

int gca_get_info(const gca_cache_t* c, gca_info_t* info) {
    if (!c || !info) return GCA_ERR_INVALID_ARG;
    info->num_pages = c->num_pages;
    info->image_pages_per_frame = c->ipf;
    info->frames = c->T;
    info->full_frames = (int)c->image_pages.size();
    info->resident_tokens = (long long)c->ftok * (long long)c->image_pages.size() +
                            (long long)c->keep * c->T;
    info->k_pool = c->kpool;
    info->v_pool = c->vpool;
    info->pool_bytes = c->pool_bytes;
    info->scratch_bytes = c->ws_slots * kTileRows * (gca::kHeadDim + 1) * sizeof(float);
    info->kernel_launches = c->launches;
    return GCA_OK;
}

int gca_device_status(gca_cache_t* c, int32_t* status_out, int32_t clear) {
    if (!c || !status_out) return GCA_ERR_INVALID_ARG;
    *status_out = *(volatile int*)c->h_status;
    if (clear) *(volatile int*)c->h_status = 0;
    return GCA_OK;
}

int gca_selftest_bounded_wait(gca_cache_t* c, int32_t timeout_ms, int32_t* status_out) {
    if (!c || !status_out || timeout_ms < 1 || timeout_ms > 10000) return GCA_ERR_INVALID_ARG;
    if (c->host_only) return GCA_ERR_UNSUPPORTED;
    DeviceGuard guard(c->device);
    if (gca::launch_bounded_wait_selftest(c->d_status, (unsigned long long)timeout_ms * 1000000ull, 0) != cudaSuccess ||
        cudaDeviceSynchronize() != cudaSuccess) {
        cudaGetLastError();
        return GCA_ERR_CUDA;
    }
    *status_out = *(volatile int*)c->h_status;
    return GCA_OK;
}

int gca_attend(gca_cache_t* c, int32_t layer, const void* q, int32_t F, void* out, float* lse,
               void* stream) {
    Range range("gca_attend");
    if (!c || !q || !out) return GCA_ERR_INVALID_ARG;
    if (!placed(q, 16) || !placed(out, 16) || !placed(lse, 4)) return GCA_ERR_INVALID_ARG;
    if (c->host_only) return GCA_ERR_UNSUPPORTED;
    const gca_config_t& g = c->cfg;
    if (layer < 0 || layer >= g.num_layers) return GCA_ERR_INVALID_ARG;
    if (F < 1 || F > g.max_query_frames) return GCA_ERR_INVALID_ARG;
    if (F > c->T || c->layer_frames[layer] != c->T) return GCA_ERR_STATE;
    if (int s = check_status(c)) return s;
    DeviceGuard guard(c->device);
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    cudaStream_t ex;
    if (!begin_call(c, st, on_host(q) && on_host(out) && (!lse || on_host(lse)), &ex)) return GCA_ERR_CUDA;
    // walk list: rebuilt and uploaded when the page table or the block changed
    if (c->up_version != c->version || c->up_F != F) {
        std::vector<gca_page_entry_t> w;
        if (!build_walk(c, F, w)) return end_call(c, st, ex, GCA_ERR_STATE);
        if (int e = upload_walk(c, w, c->d_walk, ex)) return end_call(c, st, ex, e);
        c->up_version = c->version;
        c->up_F = F;
        c->up_n = (int)w.size();
    }
    return end_call(c, st, ex, run_attention(c, layer, q, F, c->T - F, c->d_walk, c->up_n, out, lse, ex, st));
}

int gca_frame_attention(gca_cache_t* c, int32_t layer, const void* q, const void* k, const void* v,
                        void* out, float* lse, void* stream) {
    Range range("gca_frame_attention");
    if (!c || !q || !k || !v || !out) return GCA_ERR_INVALID_ARG;
    if (!placed(q, 16) || !placed(k, 16) || !placed(v, 16) || !placed(out, 16) || !placed(lse, 4))
        return GCA_ERR_INVALID_ARG;
    if (c->host_only) return GCA_ERR_UNSUPPORTED;
    if (layer < 0 || layer >= c->cfg.num_layers) return GCA_ERR_INVALID_ARG;
    if (int s = check_status(c)) return s;
    DeviceGuard guard(c->device);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaStream_t ex;
    if (!begin_call(c, st, on_host(q) && on_host(k) && on_host(v) && on_host(out) && (!lse || on_host(lse)), &ex))
        return GCA_ERR_CUDA;
    CUtensorMap fk{}, fv{};
    bool direct = false;
    if (int e = stage_transient(c, layer, k, v, 0, ex, &fk, &fv, &direct)) return end_call(c, st, ex, e);
    int rc = run_attention(c, layer, q, 1, 0, c->d_walk_f, c->tpf, out, lse, ex, st, direct ? &fk : nullptr,
                           direct ? &fv : nullptr);
    if (direct && rc == GCA_OK && cudaEventRecord(c->kv_free, ex) != cudaSuccess) rc = GCA_ERR_CUDA;
    return end_call(c, st, ex, rc);
}

int gca_frame_attention_batch(gca_cache_t* c, int32_t layer, int32_t num_frames, const void* q, const void* k,
                              const void* v, void* out, float* lse, void* stream) {
    Range range("gca_frame_attention_batch");
    if (!c || !q || !k || !v || !out || num_frames < 1) return GCA_ERR_INVALID_ARG;
    if (c->host_only) return GCA_ERR_UNSUPPORTED;
    const gca_config_t& g = c->cfg;
    if (layer < 0 || layer >= g.num_layers) return GCA_ERR_INVALID_ARG;
    if (!placed(q, 16) || !placed(k, 16) || !placed(v, 16) || !placed(out, 16) || !placed(lse, 4))
        return GCA_ERR_INVALID_ARG;
    if (int s = check_status(c)) return s;
    const size_t fb = (size_t)c->Lq * g.num_heads * gca::kHeadDim * c->elem;
    const size_t lb = (size_t)c->Lq * g.num_heads * sizeof(float);
    auto at = [](const void* base, size_t off) { return static_cast<const char*>(base) + off; };
    const bool batched = g.dtype == GCA_DTYPE_BF16 && g.rope == GCA_ROPE_NONE && !on_host(q) && !on_host(k) &&
                         !on_host(v) && !on_host(out) && (!lse || !on_host(lse));
    if (!batched) {
        // host tensors (staged per frame), an fp32 cache or RoPE (K copied and
        // rotated into the transient pages): one frame per launch
        for (int f = 0; f < num_frames; ++f)
            if (int rc = gca_frame_attention(c, layer, at(q, f * fb), at(k, f * fb), at(v, f * fb),
                                             const_cast<char*>(at(out, f * fb)),
                                             lse ? (float*)const_cast<char*>(at(lse, f * lb)) : nullptr, stream))
                return rc;
        return GCA_OK;
    }
    DeviceGuard guard(c->device);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaStream_t ex;
    if (!begin_call(c, st, false, &ex)) return GCA_ERR_CUDA;   // device tensors: the caller's stream order
    const int ppf = (ceil_div(c->Lq, kTileRows) + 1) / 2;    // tile pairs per frame
    for (int f0 = 0; f0 < num_frames; f0 += kMaxBatch) {
        const int n = std::min(kMaxBatch, num_frames - f0);
        CUtensorMap fk{}, fv{};
        if (!encode_frame_map(c, &fk, at(k, f0 * fb), n) || !encode_frame_map(c, &fv, at(v, f0 * fb), n))
            return GCA_ERR_CUDA;
        gca::AttendParams p{};
        p.walk = c->d_walk_b;
        p.nwalk = c->tpf;
        p.q = at(q, f0 * fb);
        p.out = const_cast<char*>(at(out, f0 * fb));
        p.lse = lse ? (float*)const_cast<char*>(at(lse, f0 * lb)) : nullptr;
        p.R = n * c->Lq;
        p.H = g.num_heads;
        p.Lq = c->Lq;
        p.first_query_frame = 0;
        p.rule = {g.num_anchor, g.window, c->keep, g.anchor_block ? 1 : 0};
        p.scale = c->scale;
        p.scale_log2 = c->scale * 1.4426950408889634f;
        p.layer = layer;
        p.num_pages = c->num_pages;
        p.P = c->P;
        p.status = c->d_status;
        p.ws_o = c->ws_o;
        p.ws_lse = c->ws_lse;
        p.rope = c->rope();
        // one CTA per (frame, tile pair, head): a frame's heads are a few pages
        // each, so none is split and no partial or merge is needed
        p.ppf = ppf;
        p.QT = n * 2 * ppf;
        p.W = g.num_heads;
        p.seg = c->tpf;
        p.merge_cnt = c->merge_cnt;
        p.epoch = ++c->epoch;
        p.frame_page0 = c->num_regular;
        if (gca::launch_attend_sm100(c->tmK, c->tmV, fk, fv, p, ex) != cudaSuccess) {
            cudaGetLastError();
            return GCA_ERR_CUDA;
        }
        c->launches += 1;
    }
    return GCA_OK;
}

int gca_attend_transient(gca_cache_t* c, int32_t layer, const void* q, const void* k, const void* v,
                         void* out, float* lse, void* stream) {
    Range range("gca_attend_transient");
    if (!c || !q || !k || !v || !out) return GCA_ERR_INVALID_ARG;
    if (!placed(q, 16) || !placed(k, 16) || !placed(v, 16) || !placed(out, 16) || !placed(lse, 4))
        return GCA_ERR_INVALID_ARG;
    if (c->host_only) return GCA_ERR_UNSUPPORTED;
    const gca_config_t& g = c->cfg;
    if (layer < 0 || layer >= g.num_layers) return GCA_ERR_INVALID_ARG;
    if (c->layer_frames[layer] != c->T) return GCA_ERR_STATE;
    if (int s = check_status(c)) return s;
    DeviceGuard guard(c->device);
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    // The frame reads the cache as the latest keyframe t = T-1 does (query
    // frame index t: its window and every summary), plus its own S+M tokens,
    // which the walk list carries as full-frame pages of frame t.  With no
    // keyframe yet it reads only itself.
    const int i = c->T > 0 ? c->T - 1 : 0;
    cudaStream_t ex;
    if (!begin_call(c, st, on_host(q) && on_host(k) && on_host(v) && on_host(out) && (!lse || on_host(lse)), &ex))
        return GCA_ERR_CUDA;
    if (c->tup_version != c->version) {
        std::vector<gca_page_entry_t> w;
        if (c->T > 0 && !build_walk(c, 1, w)) return end_call(c, st, ex, GCA_ERR_STATE);
        for (int s = 0; s < c->tpf; ++s) {
            const int first = s * c->P;
            w.push_back({c->num_regular + s, GCA_PAGE_IMAGE, i, first, std::min(c->P, c->Lq - first)});
        }
        if (int e = upload_walk(c, w, c->d_walk_t, ex)) return end_call(c, st, ex, e);
        c->tup_version = c->version;
        c->tup_n = (int)w.size();
    }

    CUtensorMap fk{}, fv{};
    bool direct = false;
    if (int e = stage_transient(c, layer, k, v, i, ex, &fk, &fv, &direct)) return end_call(c, st, ex, e);
    int rc = run_attention(c, layer, q, 1, i, c->d_walk_t, c->tup_n, out, lse, ex, st, direct ? &fk : nullptr,
                           direct ? &fv : nullptr);
    if (direct && rc == GCA_OK && cudaEventRecord(c->kv_free, ex) != cudaSuccess) rc = GCA_ERR_CUDA;
    return end_call(c, st, ex, rc);
}
}  // extern "C"
