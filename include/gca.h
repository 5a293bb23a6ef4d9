/*
 * gca.h — C ABI of the B200 Geometric Context Attention (GCA) hot path.
 *
 * GCA is the cross-frame attention of the Geometric Context Transformer
 * (LingBot-Map).  Each new frame carries M image-patch tokens and S = 6 summary
 * tokens (1 camera, 1 anchor, 4 register; paper digest §2.3).  Its queries
 * attend to three key sets (paper digest §2.2 frame-type table and §2.5
 * attention-mask table):
 *   (a) the n anchor frames, all tokens;
 *   (b) the k most recent frames (the pose-reference window, current frame
 *       included), all tokens;
 *   (c) the trajectory memory: only the S summary tokens of every older frame.
 * The KV cache behind it is paged (news article, inference paragraph; code
 * walkthrough §3.4) and holds M*min(T, n+k) + S*T tokens after T frames
 * (paper digest §2.4: M(n+k) + 6T).
 *
 * Library-owned state: the page pools (per layer K and V,
 * [num_pages][H][page_size][D]), one page table shared by all layers, and the
 * device copy of the walk list.  Caller-owned: every pointer passed to a call.
 *
 * Pointers: q, k, v, out and lse may be device pointers or host pointers
 * (pinned or pageable).  Host inputs are staged through library device
 * buffers by cudaMemcpyAsync on library copy streams; host outputs are written
 * to library device buffers and copied back the same way.  The stream argument
 * waits for those copies, so the caller synchronises the stream before
 * reading a host output.  Device pointers must stay valid until the stream has
 * consumed them, and start on a 16-byte boundary (lse: 4-byte), as every
 * allocation does: the kernels move 16-byte vectors, and a device pointer off
 * that boundary is refused with GCA_ERR_INVALID_ARG before anything runs.
 *
 * A call whose pointer arguments are ALL in host memory does not wait for
 * earlier work on the stream: its kernels follow the cache's earlier calls
 * only, on a library stream, so one call's copy back overlaps the next call's
 * kernels (the stream still waits for the call).  Its host inputs are read
 * after the call is made: the caller fills them before the call (not with
 * work queued on the stream) and leaves them unchanged until the stream has
 * completed the call.  Any other call (at least one device pointer) runs in
 * the stream's order.
 *
 * Streams: every GPU step is asynchronous on the stream argument (a
 * cudaStream_t; NULL = legacy default stream).  Calls on one cache must be
 * ordered on one stream (or externally synchronised): they share the walk-list
 * buffer and the scratch space.
 *
 * Tensor layouts (row-major, contiguous, dtype of the cache):
 *   frame tensors  [S+M][H][D]   summary tokens first (camera, anchor,
 *                                registers), then the M image tokens;
 *   all-layer form [L][S+M][H][D];
 *   query block    [F][S+M][H][D] for the F most recent frames;
 *   lse            [F][S+M][H] float32, natural logarithm.
 *
 * Errors: every call returns a gca_status; on error no state changes unless
 * stated.  GCA_ERR_DEVICE_CHECK reports that a kernel of this cache raised its
 * device status word (a bounded wait that ran out, or an index check); read it
 * with gca_device_status.
 */
#ifndef GCA_H_
#define GCA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GCA_ALL_LAYERS (-1)
#define GCA_HOST_ONLY (-1)   /* gca_cache_create device: the page table alone */

typedef enum {
    GCA_OK = 0,
    GCA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, bad layer index        */
    GCA_ERR_CAPACITY = 2,      /* page pool or max_frames exhausted              */
    GCA_ERR_STATE = 3,         /* call out of order (see each call)              */
    GCA_ERR_UNSUPPORTED = 4,   /* dtype, head_dim or page size not built         */
    GCA_ERR_CUDA = 5,          /* a CUDA runtime call failed                     */
    GCA_ERR_DEVICE_CHECK = 6   /* a kernel raised the device status word         */
} gca_status;

typedef enum { GCA_DTYPE_BF16 = 0, GCA_DTYPE_F32 = 1 } gca_dtype;

/* What a frame keeps once it leaves the window (its trajectory memory):
 *   SUMMARY  all S special tokens (GCA; paper digest §2.2);
 *   CAMERA   only special token 0, the camera token (the camera-only cache
 *            option of code walkthrough §3.4);
 *   NONE     nothing: with num_anchor = 0 this is the sliding-window mask of
 *            the news article's mask figure (c).
 * The special tokens a frame does not keep are stored with its image tokens
 * and leave the cache with them. */
typedef enum { GCA_MEMORY_SUMMARY = 0, GCA_MEMORY_CAMERA = 1, GCA_MEMORY_NONE = 2 } gca_memory;

/* Position encoding applied inside the library (news article, video RoPE
 * ablation; paper digest §2.7, a timestamp on the summary tokens; code
 * walkthrough §3.1, enable_3d_rope):
 *   NONE  q and k are used as given (already encoded by the caller);
 *   3D    rotary encoding (RoFormer) over time t, patch row y and patch column
 *         x: head dims 0..23 rotate with t, 24..43 with y, 44..63 with x; in
 *         each part of d dims, pair (2i, 2i+1) turns by pos * base^(-2i/d).
 *         Image token m of frame t sits at (t, m / grid_w, m % grid_w), the
 *         frame's special tokens at (t, 0, 0); t is the frame's index in the
 *         cache.  gca_append_frame rotates K as it stores it (the pools hold
 *         rotated keys, in the cache dtype), the attention calls rotate q as
 *         they load it; v is not rotated.  A non-keyframe
 *         (gca_attend_transient) takes the latest keyframe's t; intra-frame
 *         attention uses t = 0 (only differences of positions matter). */
typedef enum { GCA_ROPE_NONE = 0, GCA_ROPE_3D = 1 } gca_rope;
typedef enum { GCA_PAGE_IMAGE = 0, GCA_PAGE_SUMMARY = 1 } gca_page_kind;

typedef struct gca_cache gca_cache_t;  /* opaque, library-owned */

/* Creation parameters.  They mirror the reference constructor's arguments
 * (resolution -> image_tokens, sliding window, scale frames, tokens per frame,
 * heads, head_dim, dtype, special-token count; code walkthrough §3.1, §3.4). */
typedef struct {
    int32_t num_layers;       /* L >= 1: layers with independent KV streams      */
    int32_t num_heads;        /* H >= 1                                          */
    int32_t head_dim;         /* D: 64 (bf16 and f32)                            */
    int32_t image_tokens;     /* M >= 1: image-patch tokens per frame            */
    int32_t summary_tokens;   /* S >= 1: summary tokens per frame (6 in GCT)     */
    int32_t num_anchor;       /* n >= 0: anchor ("scale") frames                 */
    int32_t window;           /* k >= 1: pose-reference window, current frame in */
    int32_t max_frames;       /* frames appended before a reset (summary space)  */
    int32_t page_size;        /* P: 64 or 128 tokens per page                    */
    int32_t dtype;            /* gca_dtype: BF16 (tcgen05 path), F32 (SIMT path) */
    int32_t anchor_block;     /* 1: the first n frames attend to each other in
                                 full (one joint block, code walkthrough §3.2)  */
    int32_t max_query_frames; /* F_max >= 1: largest query block of gca_attend   */
    int32_t frame_slack;      /* extra full frames of page space (>= 0)          */
    float softmax_scale;      /* 0 selects 1/sqrt(D)                             */
    int32_t trajectory_memory; /* gca_memory; 0 (SUMMARY) is GCA                 */
    int32_t rope;             /* gca_rope: 3D rotary position encoding of Q, K   */
    int32_t rope_grid_w;      /* patch columns of the image-token grid (0: M)    */
    float rope_base;          /* rotary base (0 selects 10000)                   */
} gca_config_t;

/* One entry of the walk list (the pages gca_attend reads, in order).  Below,
 * s_k is the number of special tokens a frame keeps (S, 1 or 0 by
 * trajectory_memory) and M' = M + S - s_k the tokens of a full frame's image
 * pages (its unkept special tokens, then its M image tokens).
 * Image page: frame = owning frame, first = index of slot 0 among that frame's
 * M' image-page tokens.  Summary page: first = summary-stream index of slot 0
 * (kept token s of frame t has stream index s_k*t+s), frame = first / s_k.
 * n_valid = tokens stored in the page. */
typedef struct {
    int32_t page_id;
    int32_t kind;             /* gca_page_kind */
    int32_t frame;
    int32_t first;
    int32_t n_valid;
} gca_page_entry_t;

/* Sizes and pool addresses, for tests and tools. */
typedef struct {
    int32_t num_pages;        /* pool pages per layer                            */
    int32_t image_pages_per_frame;
    int32_t frames;           /* T: frames opened since create / reset           */
    int32_t full_frames;      /* frames still holding their image pages          */
    int64_t resident_tokens;  /* M' * full_frames + s_k * T                      */
    void* k_pool;             /* device: [L][num_pages][H][P][D] of dtype        */
    void* v_pool;
    size_t pool_bytes;        /* bytes of one pool (all layers)                  */
    size_t scratch_bytes;     /* device scratch owned by the cache               */
    int64_t kernel_launches;  /* kernels this cache has launched since create    */
} gca_info_t;

/* Create a cache on CUDA device `device`.  Allocates both pools:
 * num_pages = (n + k + max_query_frames + frame_slack) * ceil(M'/P)
 *           + ceil(s_k * max_frames / P) pages the allocator hands out,
 *           + ceil((S+M) / P)            transient pages after them
 *                                        (gca_attend_transient), per layer.
 * device = GCA_HOST_ONLY creates the page table alone, with no device state:
 * gca_append_frame (k and v may be NULL; nothing is copied), evict, reset,
 * get_layout, token_slot, get_info and device_status behave as on a device;
 * the attention calls and the self-test return UNSUPPORTED.  It lets a host
 * without a GPU check the page table.
 * Errors: INVALID_ARG (non-positive sizes, null out, no such device),
 * UNSUPPORTED (head_dim != 64, page_size not 64/128, unknown dtype,
 * ceil((S+M)/P) > 128), CUDA (allocation). */
int gca_cache_create(const gca_config_t* cfg, int device, gca_cache_t** out);

/* Free everything the cache owns.  The caller must have synchronised the
 * streams that used it.  Null is accepted. */
int gca_cache_destroy(gca_cache_t* cache);

/* Append one frame's K and V (code walkthrough §2: each step adds the new
 * frame's M+S tokens).  layer == GCA_ALL_LAYERS or 0 opens frame T: the
 * allocator takes a summary page if the frame's s_k kept tokens start a new
 * one, then ceil(M'/P) image pages, smallest free page id first.  With
 * GCA_ALL_LAYERS k and v are [L][S+M][H][D] and every layer is written in one
 * launch; otherwise they are [S+M][H][D] for that layer, and layers 1..L-1
 * must then append the open frame once each.  *frame_index_out (nullable)
 * receives the frame index.  Errors: CAPACITY (no pages or max_frames reached;
 * nothing changes), STATE (layer > 0 with no open frame for it, or layer 0 /
 * ALL while another layer still misses the open frame). */
int gca_append_frame(gca_cache_t* cache, int32_t layer, const void* k, const void* v,
                     int64_t* frame_index_out, void* stream);

/* Compressing eviction (code walkthrough §2; paper-to-code article §2.3):
 * after frame t, every non-anchor frame f <= t-k that still holds image pages
 * returns them to the free set.  Its s_k kept tokens stay in the summary
 * stream, so no bytes move.  Host-only, no stream.  *frames_evicted_out (nullable)
 * receives the number of frames reduced to summary tokens. */
int gca_evict_to_summary(gca_cache_t* cache, int32_t* frames_evicted_out);

/* GCA attention for one layer (paper digest §2.5): for the query block of the
 * F = num_query_frames most recent frames, q [F][S+M][H][D], query frame i
 * attends to
 *   every kept special token (s < s_k) of frames j <= i,
 *   every other token of frames j <= i with j < n or j >= i-k+1,
 *   and, with anchor_block, every token of frames j < n when i < n,
 * with softmax(scale * q.k) over those keys, fp32 accumulation.  out is
 * [F][S+M][H][D] in the cache dtype; lse (nullable) is [F][S+M][H] float32,
 * natural log.  Frames needed by the block must not have been evicted: call
 * gca_evict_to_summary after attending with a block.  Errors: STATE (layer has
 * not appended frame T-1, F > T, or a needed frame was evicted),
 * INVALID_ARG (F < 1 or F > max_query_frames), DEVICE_CHECK. */
int gca_attend(gca_cache_t* cache, int32_t layer, const void* q, int32_t num_query_frames,
               void* out, float* lse, void* stream);

/* Non-keyframe step for one layer (code walkthrough §3.2, keyframe_interval;
 * paper digest §5.1, keyframe selection): a frame that is not a keyframe is
 * predicted like any other, but its K and V never enter the cache.  Its
 * queries attend to every token the cache holds for `layer` — what the latest
 * keyframe t = T-1 reads as a single query frame (anchors, its window, every
 * summary token) — and to the frame's own S+M tokens (bidirectional), with
 * softmax(scale * q.k) and fp32 accumulation.  With no keyframe yet (T = 0) it
 * reads only its own tokens.
 * q, k, v: [S+M][H][D] of this layer (summary tokens first), device or host
 * memory; out [S+M][H][D] in the cache dtype; lse (nullable) [S+M][H]
 * float32, natural log.  For a bf16 cache without RoPE the attention kernel
 * reads k and v where they are (one launch; host tensors are staged first);
 * otherwise they are copied into ceil((S+M)/P) transient pages of this layer
 * (past the allocator's pages), which the next call for the layer reuses.
 * The page table, frame count and eviction state do not change, so calls for
 * one layer must be ordered (one stream).
 * Errors: STATE (layer has not appended frame T-1, or a frame the latest
 * keyframe needs was evicted), INVALID_ARG, DEVICE_CHECK. */
int gca_attend_transient(gca_cache_t* cache, int32_t layer, const void* q, const void* k,
                         const void* v, void* out, float* lse, void* stream);

/* Intra-frame attention of one frame for one layer (paper digest §3: the
 * model alternates intra-frame attention with the cross-frame GCA layers;
 * news article, pipeline figure): every token of the frame attends to every
 * token of the same frame, bidirectionally, softmax(scale * q.k), fp32
 * accumulation; no other frame is read.  q, k, v, out: [S+M][H][D] in the
 * cache dtype, device or host memory; lse (nullable) [S+M][H] float32.  k and
 * v are read like gca_attend_transient's (in place for a bf16 cache without
 * RoPE, else through the layer's transient pages); the cache's page table and
 * frames are neither read nor changed.  Errors: INVALID_ARG, DEVICE_CHECK. */
int gca_frame_attention(gca_cache_t* cache, int32_t layer, const void* q, const void* k,
                        const void* v, void* out, float* lse, void* stream);

/* Intra-frame attention of num_frames frames for one layer, each frame
 * attending only to its own tokens, as gca_frame_attention does for one.
 * q, k, v, out: [F][S+M][H][D] (F = num_frames >= 1) in the cache dtype;
 * lse (nullable) [F][S+M][H] float32.  For a bf16 cache without RoPE and
 * device tensors, up to 64 frames go in one launch with one CTA per (frame,
 * query-tile pair, head), k and v read in place; otherwise (host tensors, an
 * fp32 cache, RoPE) each frame is one gca_frame_attention call.  The cache's
 * page table and frames are neither read nor changed.
 * Errors: INVALID_ARG, DEVICE_CHECK, CUDA. */
int gca_frame_attention_batch(gca_cache_t* cache, int32_t layer, int32_t num_frames, const void* q,
                              const void* k, const void* v, void* out, float* lse, void* stream);

/* Back to the creation state (windowed mode: state is reset at each window
 * start; code walkthrough §3.3).  Page tables become identical to a fresh
 * cache's; pool bytes are left as they are and never read before rewritten. */
int gca_reset(gca_cache_t* cache);

/* The walk list gca_attend would read for a block of F most recent frames:
 * image pages of the full frames the block may see (ascending frame, page
 * order), then every summary page in stream order.  Writes min(n, cap)
 * entries to out (nullable when cap == 0) and the full count to *n_out. */
int gca_get_layout(const gca_cache_t* cache, int32_t num_query_frames,
                   gca_page_entry_t* out, int32_t cap, int32_t* n_out);

/* (page id, slot) of token slot tau of frame `frame` (tau < s_k: summary
 * stream, else the frame's image pages).  Errors: INVALID_ARG (frame not
 * appended, tau out of range), STATE (the frame's image pages were evicted
 * and tau >= s_k). */
int gca_token_slot(const gca_cache_t* cache, int32_t frame, int32_t tau,
                   int32_t* page_id_out, int32_t* slot_out);

/* The per-frame mask the attention kernels apply (paper digest §2.5, with the
 * cache's n, k, s_k and anchor_block): how many tokens of walk-list entry
 * *entry query frame `query_frame` may see.  The visible tokens of a page are
 * always its first *prefix_out slots, so one integer per (frame, page) is the
 * whole mask.  For tests and tools; works on host-only caches.
 * Errors: INVALID_ARG (null pointer, negative query frame). */
int gca_visible_prefix(const gca_cache_t* cache, const gca_page_entry_t* entry,
                       int32_t query_frame, int32_t* prefix_out);

int gca_get_info(const gca_cache_t* cache, gca_info_t* info);

/* Device status word of the cache's kernels (0 = clean) as seen now; it is
 * complete once the streams that ran them are synchronised.  clear != 0
 * resets it. */
int gca_device_status(gca_cache_t* cache, int32_t* status_out, int32_t clear);

/* Failure-detection self-test: runs the kernels' bounded mbarrier wait on a
 * barrier phase that nothing completes, with a deadline of timeout_ms (1 ..
 * 10000).  The wait gives up, raises the cache's device status word and the
 * kernel returns; the call synchronises the device and writes the status word
 * (1 = a wait ran out) to *status_out.  Clear it with gca_device_status(.., 1)
 * before further calls on the cache. */
int gca_selftest_bounded_wait(gca_cache_t* cache, int32_t timeout_ms, int32_t* status_out);

/* Static text of a status code. */
const char* gca_status_string(int status);

/* GCA attention over caller-owned pages, allocating no device memory.  The
 * paper has no counterpart; it serves callers that cannot call cudaMalloc:
 * a host framework whose caching allocator owns the device memory, or a
 * real-time loop that must not make a call that can synchronise the device.
 * Computes what gca_attend computes, with the bf16 tcgen05 kernel, for pools
 * k_pool/v_pool laid out [num_layers][num_pages][num_heads][page_size][64]
 * bf16 (device), a walk list of nwalk gca_page_entry_t (host or device; the
 * entries gca_get_layout returns), q/out [F][tokens_per_frame][H][64] bf16
 * (device) whose row 0 belongs to frame first_query_frame, lse [F][Lq][H]
 * float32 (device, nullable) and status (device int, nullable: raised like
 * the cache's status word).  summary_tokens is the number of special tokens
 * each frame keeps in the summary stream (s_k: S, 1 or 0 by the cache's
 * trajectory_memory; 0 <= s_k <= tokens_per_frame).
 * Checks before any launch (INVALID_ARG): every device buffer must lie inside
 * its allocation for the sizes given (the pools for num_layers * num_pages
 * pages, q and out for F * tokens_per_frame rows, lse, status, a device walk
 * list); a host walk list must hold page ids in [0, num_pages), n_valid in
 * [0, page_size] and a known kind.  A device walk list is checked by the
 * kernel, which raises *status on a bad page id.  With status = NULL a
 * device-side failure (a bad page id in a device walk list, a bounded wait
 * that ran out) is not reported to the caller, and out may be left unwritten.
 * A real-time caller should pass the walk list in device or pinned host
 * memory: a pageable host list is staged by a copy that can block the host.
 * Scratch (split-head partials and their counters, a device copy of the walk
 * list) lives in one static device array of 18 MiB per GPU: at most 32768
 * walk entries and 512 partial tiles of 128 query rows
 * (ceil(F*Lq/128) * H <= 512), else GCA_ERR_CAPACITY.  The first call on a
 * device looks up the array's address (call it before any stream capture);
 * calls whose GPU work overlaps share the array and race. */
int gca_attend_pages_noalloc(const void* k_pool, const void* v_pool, int32_t num_layers,
                             int32_t num_pages, int32_t num_heads, int32_t page_size,
                             int32_t layer, const gca_page_entry_t* walk, int32_t nwalk,
                             const void* q, int32_t num_query_frames, int32_t tokens_per_frame,
                             int32_t first_query_frame, int32_t num_anchor, int32_t window,
                             int32_t summary_tokens, int32_t anchor_block, float softmax_scale,
                             void* out, float* lse, int32_t* status, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* GCA_H_ */
