// Internal declarations shared by the host code and the kernels of libgca.
#pragma once

#include <climits>
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gca {

constexpr int kMaxImagePages = 128;     // image pages per frame (M <= 128 * P)
constexpr int kHeadDim = 64;

// Device walk-list entry: x = page id, y = tokens stored, z = first index
// (image: among the frame's image tokens; summary: summary-stream index),
// w = owning frame for an image page, -1 for a summary page.
using WalkEntry = int4;

// Visibility of one walk-list page to query frame i, as a prefix length: keys
// 0..nvis-1 of the page are visible, the rest are not.  Every GCA mask is a
// prefix of each page: an image page belongs to one frame and is all-or-none;
// a summary page holds frames in stream order, so the visible tokens (frames
// <= i) are its leading slots.
struct MaskRule {
    int n;             // anchor frames
    int k;             // window frames (current frame included)
    int S;             // summary tokens per frame
    int anchor_block;  // anchors see each other in full
};

__host__ __device__ inline int visible_prefix(const MaskRule& r, int4 e, int i) {
    if (e.w >= 0) {
        const int j = e.w;
        const bool vis = (r.anchor_block && i < r.n && j < r.n) ||
                         (j <= i && (j < r.n || j >= i - r.k + 1));
        return vis ? e.y : 0;
    }
    const int lim = (r.anchor_block && i < r.n) ? r.S * r.n : r.S * (i + 1);
    int v = lim - e.z;
    v = v < 0 ? 0 : v;
    return v < e.y ? v : e.y;
}

// 3D rotary encoding tables (cos, sin) of the 32 dim pairs of a head: pairs
// 0..11 turn with the frame's time index (rope_t[t * 12 + i]), pairs 12..31
// with the token's patch row and column (rope_sp[u * 20 + i - 12], u = the
// token's index in its frame, special tokens first).
constexpr int kRopeTPairs = 12;
constexpr int kRopeSpPairs = 20;

struct RopeTables {
    const float2* t;          // [max_t][12], or null: no rotation
    const float2* sp;         // [S+M][20]
    int max_t;                // rows of t
};

#ifdef __CUDACC__
// (cos, sin) of dim pair i (0..31) for token u of a frame at time index t
__device__ __forceinline__ float2 rope_cs(const RopeTables& r, int t, int u, int i) {
    t = t < r.max_t ? t : r.max_t - 1;
    return i < kRopeTPairs ? r.t[t * kRopeTPairs + i] : r.sp[u * kRopeSpPairs + (i - kRopeTPairs)];
}
// (a, b) -> (a cos - b sin, a sin + b cos)
__device__ __forceinline__ void rope_rotate(float& a, float& b, float2 cs) {
    const float a2 = fmaf(a, cs.x, -b * cs.y);
    b = fmaf(a, cs.y, b * cs.x);
    a = a2;
}
#endif

struct AppendParams {
    const void* k;            // [nlayers][Lq][H][D]
    const void* v;
    void* kpool;              // [L][num_pages][H][P][D]
    void* vpool;
    int layer0, nlayers;
    int Lq, S, M, H, P, num_pages, elem_bytes;
    int frame;
    int sum_seq0;             // summary page sequence number of this frame's token 0
    int sum_page[2];          // page ids of summary sequences sum_seq0, sum_seq0+1
    int new_sum_seq;          // summary sequence opened by this frame, -1 if none
    int img_pages[kMaxImagePages];
    int sms;                  // SMs of the device (grid sizing)
    RopeTables rope;          // K of tensor 0 is rotated when rope.t is set
    int rope_t;               // time index of the frame
};

struct AttendParams {
    const WalkEntry* walk;
    int nwalk;
    const void* q;            // [R][H][D]
    void* out;                // [R][H][D]
    float* lse;               // [R][H] natural log, nullable
    int R, H, Lq;
    int first_query_frame;    // frame of row 0
    MaskRule rule;
    float scale_log2;         // softmax scale * log2(e)
    float scale;              // softmax scale
    int layer, num_pages, P;
    // split of the head-major (head, walk entry) stream over W workers
    int QT, W, seg;
    float* ws_o;              // [QT*(W+H-1)][128][D] partial outputs (normalised)
    float* ws_lse;            // [QT*(W+H-1)][128] partial log2-sum-exp
    int* status;              // device status word (host-mapped)
    RopeTables rope;          // q rotated on load when rope.t is set
    // split heads: per-(query tile, head) count of finished workers, tagged
    // with the launch's epoch in the high word (no reset between launches)
    unsigned long long* merge_cnt;   // [QT][H]
    unsigned int epoch;
    // walk-list pages with id >= frame_page0 hold the query frame's own
    // tokens: they are read from the caller's [S+M][H][D] K and V through the
    // frame tensor maps (token `first` of the walk entry onwards) instead of
    // the pools.  INT_MAX when unused.
    int frame_page0;
    // batched frame attention (ppf > 0): R = F * Lq rows, F frames each with
    // ppf tile pairs; frame f's tile pairs walk only its own nwalk entries at
    // walk + f * nwalk, and its rows are frame first_query_frame + f
    int ppf;
};

// Work split of the bf16 attention kernel: `pairs` query-tile pairs times W
// workers, each worker a contiguous segment of `seg` entries of the
// head-major (head, walk entry) stream.  One wave of CTAs (pairs * W <= SMs),
// at least 4 entries per segment, W <= max_w.  A head whose walk is short
// (kShortWalk pages or fewer) is not split when one CTA per (pair, head) fits
// in a wave: splitting it costs more in pipeline fill, partial writes and the
// merge than its few pages take (one 518x378 frame: 25 us unsplit, 37 us
// split four ways).
constexpr int kShortWalk = 12;
inline void split_work(int sms, int pairs, int H, int nwalk, long long max_w, int* W, int* seg) {
    const long long total = (long long)H * nwalk;
    long long w = sms / pairs > 1 ? sms / pairs : 1;
    w = w < (total + 3) / 4 ? w : (total + 3) / 4;
    w = w < max_w ? w : max_w;
    w = w > 1 ? w : 1;
    long long s = (total + w - 1) / w;
    if (s < nwalk && nwalk <= kShortWalk && (long long)pairs * H <= sms) s = nwalk;
    *seg = (int)s;
    *W = (int)((total + s - 1) / s);
}

// launchers (return cudaError_t of the launch)
cudaError_t launch_append(const AppendParams& p, cudaStream_t s);
// tk / tv: the pools as [L * num_pages * H * P][D]; tkf / tvf: a frame's
// [S+M][H][D] K and V (read for pages >= p.frame_page0; any valid map when
// p.frame_page0 is INT_MAX)
cudaError_t launch_attend_sm100(const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tkf,
                                const CUtensorMap& tvf, const AttendParams& p, cudaStream_t s);
cudaError_t launch_bounded_wait_selftest(int* status, unsigned long long timeout_ns, cudaStream_t s);
cudaError_t launch_attend_f32(const AttendParams& p, const void* kpool, const void* vpool,
                              cudaStream_t s);

// device status codes
enum : int {
    kStatusWaitTimeout = 1,
    kStatusBadPage = 2,
};

}  // namespace gca
