// GCA attention for sm_100a: tcgen05 tensor cores, TMEM accumulators, TMA.
//
// Computes, for every query row r of the block and head h (paper digest §2.5:
// the current frame attends to anchors and window frames with all tokens and
// to the summary tokens of every earlier frame),
//     O[r,h] = softmax_u(scale * q[r,h] . k[u,h]) v[u,h]
// over the keys of the walk list that row r's frame may see.  Each walk-list
// page's visible keys are a prefix of its slots (see visible_prefix), so the
// mask is one integer per (row, page).
//
// Work split.  Query rows form pairs of 128-row tiles (256 rows per CTA).  The
// head-major stream of (head, walk entry) pairs is cut into W contiguous
// segments; CTA (pair, w) runs its two tiles over segment w.  All CTAs of a
// segment read the same K/V pages in the same order at about the same time,
// so each page comes from HBM once and from L2 for the others.  A segment that
// covers a whole head writes the final output; heads split between segments
// leave normalised partials plus their log-sum-exp, and the worker that
// finishes a split head last (a per-(tile, head) counter) combines them.
//
// Per CTA (384 threads, one CTA per SM):
//   warps 0-3 / 4-7  softmax of tile 0 / tile 1: thread t owns query row t of
//              its tile (TMEM lane t); writes its Q row into shared memory,
//              reads S rows from TMEM, online softmax in the log2 domain,
//              writes P (bf16) back over the S columns, final normalisation;
//   warp 8     TMA producer: one (page, head) K tile and V tile per stage,
//              128-byte swizzled boxes of P x 64 bf16, 4 stages;
//   warps 9/10 one MMA-issuing thread per tile (warp 9 also owns TMEM; warp
//              11 idle).  Any wait in an issuing thread stalls its tcgen05.mma
//              stream (the tensor core takes about one instruction ahead of
//              the issuer): a mbarrier wait on an already completed phase
//              costs ~200 cycles of tensor-pipe time.  With one issuer per
//              tile, each issuer's waits are covered by the other's MMAs.
//
// Three rotating S buffers.  TMEM holds three S buffers of P columns and the
// two tiles' O accumulators: 3 x 128 + 2 x 64 = 512 columns for 128-token
// pages.  QK of tile t for page j (index i = 2j + t) writes buffer i % 3.  Per
// page, tile t's issuer runs S_t(j) = Q_t K_j^T, then O_t += P_t(j-1) V_{j-1},
// so each tile's next S is computed while its softmax of the current page
// runs, and the two softmax groups work side by side instead of taking turns.
// Buffer i % 3 last held index i - 3 (the other tile), whose PV reads its P:
// the QK waits for that PV to complete (buf_free, one phase per use of the
// buffer).  Q sits in shared memory (SS-form QK), two buffers per tile, so
// the softmax warps load the next head's Q while the current head runs.
//
// A warp may start page j+1 (its S is ready) while the other warps of its
// tile finish page j, so the "P written" barrier is split by page parity:
// arrivals for page j+1 never count toward page j.
//
// Softmax: a page is exponentiated against the row's running max without
// computing the page max first.  Since relative precision does not depend on
// scale, values up to 2^64 are as good as values up to 1; a row whose page
// sum reaches 2^64 (or overflows) takes the exact path instead: page max, O
// rescaled by 2^(m_old - m_new) once the previous PV has completed (the
// page's K/V stage released by both tiles' PVs),
// exponentials recomputed.  The first page of every head always takes the
// exact path.  Scores are scaled and shifted with packed f32x2 FMAs; every
// exponential runs on the MUFU unit (ex2.approx): with this schedule the
// kernel is not MUFU-bound, and moving part of them to an FMA-pipe polynomial
// measured slower.
//
// Every wait on an mbarrier is bounded by a %globaltimer deadline; on expiry
// the thread raises the CTA abort flag and the device status word, every role
// leaves its loop, in-flight TMA loads and MMAs are drained (bounded), TMEM is
// freed and the kernel returns.
#include <cuda_bf16.h>

#include "gca_internal.h"

namespace gca {

namespace {

constexpr int kThreads = 384;               // 3 warpgroups: softmax 0, softmax 1, TMA + MMA
constexpr int kWarpTMA = 8;
constexpr int kWarpMMA = 9;
// Register split (setmaxnreg): launched at 168 per thread (384 x 168 = 64512);
// the two softmax warpgroups take 216, the producer warpgroup keeps 64:
// 256 x 216 + 128 x 64 = 63488 <= 64512.
constexpr int kRegsSoftmax = 216;
constexpr int kRegsProducer = 64;
static_assert(256 * kRegsSoftmax + 128 * kRegsProducer <= kThreads * 168, "register split");
constexpr int kStages = 4;
constexpr int kRows = 128;
constexpr uint32_t kTmemCols = 512;
constexpr unsigned long long kTimeoutNs = 2000000000ull;
template <int PAGE>
struct Layout {
    static constexpr int kTileBytes = PAGE * 128;          // PAGE x 64 bf16
    static constexpr int kStageBytes = 2 * kTileBytes;     // K then V
    static constexpr int kQBytes = 128 * 128;              // one tile's Q: 128 rows x 64 bf16, SW128
    static_assert(3 * PAGE + 128 <= (int)kTmemCols, "TMEM budget: 3 S buffers + 2 O");
    static constexpr int kNumBars = 2 * kStages + 27;
    static constexpr int kSmemBytes = kStages * kStageBytes + 4 * kQBytes + kNumBars * 8 + 16 + 1024;
};

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        "selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ unsigned long long globaltimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

struct Ctl {
    volatile int* abort;
    int* status;
};

// Bounded parity wait.  honour_abort = false is used while draining.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, Ctl c, bool honour_abort = true,
                                         unsigned long long timeout_ns = kTimeoutNs) {
    if (mbar_try(bar, parity)) return true;
    const unsigned long long t0 = globaltimer();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try(bar, parity)) return true;
        if ((it & 127u) == 0) {
            if (honour_abort && *c.abort) return false;
            if (globaltimer() - t0 > timeout_ns) {
                *c.abort = 1;
                *(volatile int*)c.status = kStatusWaitTimeout;
                __threadfence_system();
                return false;
            }
        }
    }
}


__device__ __forceinline__ void fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* tm, int x, int y,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* tm, int x, int y, int z,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(z), "r"(bar)
        : "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle (tcgen05 format:
// start >> 4 in [0,14), leading byte offset >> 4 in [16,30), stride byte
// offset >> 4 in [32,46), version 1 at [46,48), swizzle mode 2 at [61,64)).
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor, kind::f16: D f32 (bits 4-5 = 1), A and B bf16
// (bits 7-9 = 1, 10-12 = 1), B major at bit 16, N >> 3 at [17,23), M >> 4 at
// [24,29).
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// D[tmem] (+)= A[tmem] * B[smem desc]
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}" ::"r"(d),
        "r"(a), "l"(b), "r"(idesc), "r"(accumulate)
        : "memory");
}
// D[tmem] (+)= A[smem desc] * B[smem desc]; descriptors as 32-bit halves
__device__ __forceinline__ void mma_ss(uint32_t d, uint32_t a_lo, uint32_t a_hi, uint32_t b_lo,
                                       uint32_t b_hi, uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n.reg .pred p;\n.reg .b64 ad, bd;\nsetp.ne.b32 p, %6, 0;\nmov.b64 ad, {%1, %2};\n"
        "mov.b64 bd, {%3, %4};\n"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %5, p;\n}" ::"r"(d),
        "r"(a_lo), "r"(a_hi), "r"(b_lo), "r"(b_hi), "r"(idesc), "r"(accumulate)
        : "memory");
}
// D[tmem] += A[tmem] * B[smem desc]; B given as its two 32-bit halves
__device__ __forceinline__ void mma_ts_acc(uint32_t d, uint32_t a, uint32_t b_lo, uint32_t b_hi,
                                           uint32_t idesc) {
    asm volatile(
        "{\n.reg .b64 bd;\nmov.b64 bd, {%2, %3};\n"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], bd, %4, 1;\n}" ::"r"(d),
        "r"(a), "r"(b_lo), "r"(b_hi), "r"(idesc)
        : "memory");
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
        : "memory");
}

#define GCA_R8(i) "=r"(r[i + 0]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3]), \
                  "=r"(r[i + 4]), "=r"(r[i + 5]), "=r"(r[i + 6]), "=r"(r[i + 7])
#define GCA_W8(i) "r"(r[i + 0]), "r"(r[i + 1]), "r"(r[i + 2]), "r"(r[i + 3]), \
                  "r"(r[i + 4]), "r"(r[i + 5]), "r"(r[i + 6]), "r"(r[i + 7])

// 32 consecutive 32-bit TMEM columns of this thread's lane
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : GCA_R8(0), GCA_R8(8), GCA_R8(16), GCA_R8(24)
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t* r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : GCA_R8(0), GCA_R8(8)
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        GCA_W8(0), GCA_W8(8)
        : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}


// packed f32x2 arithmetic (two lanes of work per instruction)
__device__ __forceinline__ uint64_t f2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void unf2(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t fmul2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}


// ---------------------------------------------------------------------------
// ---------------------------------------------------------------------------
// the kernel: two query tiles, three rotating S buffers
// ---------------------------------------------------------------------------
// QK_t(j) (tile t, page j) writes S buffer (2j + t) % 3.  The buffer's previous
// user is QK of index 2j + t - 3, whose PV is issued before QK_t(j), so each
// tile's next S is computed while its softmax of the current page runs.
template <int PAGE, bool BATCH>
__global__ void __launch_bounds__(kThreads, 1)
attend_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
              const __grid_constant__ CUtensorMap tmKf, const __grid_constant__ CUtensorMap tmVf,
              const AttendParams p) {
    using L = Layout<PAGE>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t qbase = sbase + kStages * L::kStageBytes;     // Q[t][buf] at + (2t+buf)*kQBytes
    uint8_t* qsm = smem + kStages * L::kStageBytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(qsm + 4 * L::kQBytes);
    const uint32_t bar0 = smem_u32(bars);
    auto kv_full = [&](int s) { return bar0 + 8u * s; };
    auto kv_empty = [&](int s) { return bar0 + 8u * (kStages + s); };
    auto s_full = [&](int b) { return bar0 + 8u * (2 * kStages + b); };           // 3 buffers
    // P of tile t written for page j: p_full(t, j & 1).  One barrier per page
    // parity: a warp may start page j+1 (its S is already computed) while the
    // tile's other warps still finish page j, so its arrivals must not count
    // toward page j's phase; it cannot reach page j+2 before page j's phase
    // completed (QK_t(j+2) is issued only after PV_t(j)).
    auto p_full = [&](int t, int par) { return bar0 + 8u * (2 * kStages + 14 + 2 * t + par); };
    auto q_ready = [&](int t, int b) { return bar0 + 8u * (2 * kStages + 7 + 2 * t + b); };
    // drain(t): MMA thread t's last MMAs have completed (before TMEM is freed)
    auto drain = [&](int t) { return bar0 + 8u * (2 * kStages + 18 + t); };
    // buf_free(b): the PV that read S buffer b's P has completed, so the next
    // QK may overwrite it (the two tiles' QKs and PVs come from two threads)
    auto buf_free = [&](int b) { return bar0 + 8u * (2 * kStages + 20 + b); };
    // o_done(t): PV_t of a head's last page has completed (one phase per head)
    auto o_done = [&](int t) { return bar0 + 8u * (2 * kStages + 12 + t); };
    // fused merge of a split head: every row of the tile has written its partial
    // (mrg_all, 128 arrivals), then the tile's elected thread posts whether this
    // CTA is the head's last worker (mrg_flag, 1 arrival)
    auto mrg_all = [&](int t) { return bar0 + 8u * (2 * kStages + 23 + t); };
    auto mrg_flag = [&](int t) { return bar0 + 8u * (2 * kStages + 25 + t); };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + L::kNumBars);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* last_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);    // [2]: per tile
    const Ctl ctl{abort_flag, p.status};

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int qp = blockIdx.x;
    // batched frame attention: CTA row qp is tile pair qp % ppf of frame
    // qp / ppf, which walks only that frame's own entries
    const int bframe = BATCH ? qp / p.ppf : 0;
    const int qpl = BATCH ? qp - bframe * p.ppf : qp;
    const WalkEntry* const walk = p.walk + (BATCH ? (long long)bframe * p.nwalk : 0ll);
    const int w = blockIdx.y;
    const long long total = (long long)p.H * p.nwalk;
    const long long g0 = (long long)w * p.seg;
    const long long g1 = (g0 + p.seg < total) ? g0 + p.seg : total;
    const int J = (int)(g1 - g0);
    const int h_start = (int)(g0 / p.nwalk);
    const int e_start = (int)(g0 - (long long)h_start * p.nwalk);
    const int h_last = (int)((g1 - 1) / p.nwalk);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(kv_full(s), 1);
            mbar_init(kv_empty(s), 2);          // both tiles' PV of the stage's page
        }
        for (int b = 0; b < 3; ++b) mbar_init(s_full(b), 1);
        for (int t = 0; t < 2; ++t) {
            mbar_init(p_full(t, 0), kRows);
            mbar_init(p_full(t, 1), kRows);
            mbar_init(q_ready(t, 0), kRows);
            mbar_init(q_ready(t, 1), kRows);
            mbar_init(o_done(t), 1);
            mbar_init(mrg_all(t), kRows);
            mbar_init(mrg_flag(t), 1);
        }
        for (int t = 0; t < 2; ++t) mbar_init(drain(t), 1);
        for (int b = 0; b < 3; ++b) mbar_init(buf_free(b), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == kWarpMMA) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (warp == kWarpTMA && lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmK)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmV)) : "memory");
        if (p.frame_page0 < p.num_pages) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmKf)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmVf)) : "memory");
        }
    }
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem = *tmem_slot;
    if (warp >= 8) {
      asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsProducer));
      if (warp == kWarpTMA) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int issued = 0;
            bool ok = true;
            int h = h_start, e = e_start;
            for (int j = 0; j < J; ++j) {
                const int st = j % kStages;
                if (j >= kStages && !wait_bar(kv_empty(st), ((j / kStages) - 1) & 1, ctl)) {
                    ok = false;
                    break;
                }
                const int4 ent = __ldg(&walk[e]);
                const int page = ent.x;
                if (page < 0 || page >= p.num_pages) {
                    *abort_flag = 1;
                    *(volatile int*)p.status = kStatusBadPage;
                    ok = false;
                    break;
                }
                const uint32_t dst = sbase + st * L::kStageBytes;
                mbar_expect_tx(kv_full(st), 2 * L::kTileBytes);
                if (page >= p.frame_page0) {
                    // the frame's own tokens first .. first+PAGE-1 of head h
                    // (past the last token the box reads zeros)
                    tma_load_3d(dst, &tmKf, 0, h, ent.z, kv_full(st));
                    tma_load_3d(dst + L::kTileBytes, &tmVf, 0, h, ent.z, kv_full(st));
                } else {
                    const int y = ((p.layer * p.num_pages + page) * p.H + h) * PAGE;
                    tma_load_2d(dst, &tmK, 0, y, kv_full(st));
                    tma_load_2d(dst + L::kTileBytes, &tmV, 0, y, kv_full(st));
                }
                ++issued;
                if (++e == p.nwalk) {
                    e = 0;
                    ++h;
                }
            }
            if (!ok) {
                const int from = issued > kStages ? issued - kStages : 0;
                for (int j = from; j < issued; ++j)
                    wait_bar(kv_full(j % kStages), (j / kStages) & 1, ctl, false);
            }
        }
        __syncwarp();
      } else if (warp == kWarpMMA || warp == kWarpMMA + 1) {
        // ------------------------------------------------------------ MMA issuers
        // one thread per query tile: warp 9 issues tile 0's MMAs, warp 10 tile
        // 1's, so one thread's waits are covered by the other's MMAs
        if (lane == 0) {
            const int t = warp - kWarpMMA;
            constexpr uint32_t kIdescQK = idesc_bf16(kRows, PAGE, false);
            constexpr uint32_t kIdescPV = idesc_bf16(kRows, 64, true);
            const uint64_t kdesc0 = desc_sw128(sbase, 16, 1024);
            const uint64_t vdesc0 = desc_sw128(sbase + L::kTileBytes, L::kTileBytes, 1024);
            const uint64_t qdesc0 = desc_sw128(qbase, 16, 1024);
            constexpr uint32_t kStageStep = L::kStageBytes >> 4;
            constexpr uint32_t kQStep = L::kQBytes >> 4;
            const uint32_t kd_lo0 = (uint32_t)kdesc0, kd_hi = (uint32_t)(kdesc0 >> 32);
            const uint32_t vd_lo0 = (uint32_t)vdesc0, vd_hi = (uint32_t)(vdesc0 >> 32);
            const uint32_t qd_lo0 = (uint32_t)qdesc0 + 2 * t * kQStep, qd_hi = (uint32_t)(qdesc0 >> 32);
            const uint32_t ocol = tmem + 3 * PAGE + t * 64;
            bool ok = true;
            int hs = 0;                                  // heads started in this segment
            int e = e_start;
            bool prev_first = false, prev_last = false;
            int st = 0, prev_st = 0;
            for (int j = 0; j <= J && ok; ++j) {
                const bool live = j < J;
                const bool seg_first = live && ((j == 0) || (e == 0));
                const bool seg_last = live && ((j == J - 1) || (e == p.nwalk - 1));
                if (live) {
                    const int qb = seg_first ? (hs & 1) : ((hs - 1) & 1);
                    if (seg_first) {
                        if (!wait_bar(q_ready(t, hs & 1), (hs >> 1) & 1, ctl)) { ok = false; break; }
                        ++hs;
                    }
                    if (!wait_bar(kv_full(st), (j / kStages) & 1, ctl)) { ok = false; break; }
                    // S buffer i % 3 (i = 2j + t) was last read, as P, by the PV of index i - 3
                    const int i = 2 * j + t;
                    const int b = i % 3;
                    if (i >= 3 && !wait_bar(buf_free(b), ((i / 3) - 1) & 1, ctl)) { ok = false; break; }
                    fence_after();
                    const uint32_t kd_lo = kd_lo0 + st * kStageStep;
                    const uint32_t qd_lo = qd_lo0 + qb * kQStep;
                    const uint32_t scol = tmem + b * PAGE;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)   // 16 head dims per step: +32 bytes
                        mma_ss(scol, qd_lo + 2 * kk, qd_hi, kd_lo + 2 * kk, kd_hi, kIdescQK, kk ? 1u : 0u);
                    mma_commit(s_full(b));
                }
                if (j > 0) {
                    // O_t += P_t(j-1) V_{j-1} once the tile's softmax has written P
                    const int jj = j - 1;
                    if (!wait_bar(p_full(t, jj & 1), (jj >> 1) & 1, ctl)) { ok = false; break; }
                    fence_after();
                    const int b = (2 * jj + t) % 3;
                    const uint64_t vd = vdesc0 + prev_st * kStageStep;
                    const uint32_t vd_lo = vd_lo0 + prev_st * kStageStep;
                    const uint32_t pcol = tmem + b * PAGE;
                    mma_ts(ocol, pcol, vd, kIdescPV, prev_first ? 0u : 1u);
#pragma unroll
                    for (int kk = 1; kk < PAGE / 16; ++kk)   // 16 keys per step
                        mma_ts_acc(ocol, pcol + kk * 8, vd_lo + 128 * kk, vd_hi, kIdescPV);
                    mma_commit(buf_free(b));
                    if (prev_last) mma_commit(o_done(t));
                    mma_commit(kv_empty(prev_st));
                }
                prev_first = seg_first;
                prev_last = seg_last;
                prev_st = st;
                st = (st + 1 == kStages) ? 0 : st + 1;
                if (++e == p.nwalk) e = 0;
            }
            // drain: every MMA this thread issued completes before TMEM is released
            mma_commit(drain(t));
            wait_bar(drain(t), 0, ctl, false);
        }
        __syncwarp();
      }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
        // ------------------------------------------------------------ softmax
        const int t = warp >> 2;
        const int quarter = warp & 3;
        const int rl = quarter * 32 + lane;
        const int row_l = (qpl * 2 + t) * kRows + rl;
        const int row = BATCH ? bframe * p.Lq + row_l : row_l;
        const bool valid = BATCH ? row_l < p.Lq : row < p.R;
        const int qframe = p.first_query_frame + (BATCH ? bframe : (valid ? row / p.Lq : 0));
        const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
        const uint32_t t_o = tmem + lane_base + 3 * PAGE + t * 64;
        const float sl2 = p.scale_log2;
        const __nv_bfloat16* qg = static_cast<const __nv_bfloat16*>(p.q);

        // Q of head h into Q buffer qb of this tile (K-major, 128-byte swizzle)
        auto load_q = [&](int h, int qb) {
            uint32_t r[32];
            if (valid) {
                const uint4* src = reinterpret_cast<const uint4*>(qg + ((long long)row * p.H + h) * 64);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint4 v = __ldg(src + i);
                    r[4 * i + 0] = v.x;
                    r[4 * i + 1] = v.y;
                    r[4 * i + 2] = v.z;
                    r[4 * i + 3] = v.w;
                }
                if (p.rope.t) {
                    const int u = row % p.Lq;
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        __nv_bfloat162 b2 = *reinterpret_cast<__nv_bfloat162*>(&r[i]);
                        float a = __low2float(b2), b = __high2float(b2);
                        rope_rotate(a, b, rope_cs(p.rope, qframe, u, i));
                        r[i] = pack_bf16(a, b);
                    }
                }
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) r[i] = 0u;
            }
            uint8_t* qrow = qsm + (2 * t + qb) * L::kQBytes + rl * 128;
#pragma unroll
            for (int i = 0; i < 8; ++i)
                *reinterpret_cast<uint4*>(qrow + ((i ^ (rl & 7)) * 16)) =
                    make_uint4(r[4 * i], r[4 * i + 1], r[4 * i + 2], r[4 * i + 3]);
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            mbar_arrive(q_ready(t, qb));
        };
        auto all_ok = [&](bool ok) { return __all_sync(0xffffffffu, ok); };

        float m_run = -INFINITY, l_run = 0.f;
        int hs = 0;                                    // heads started
        int hd = 0;                                    // heads finished (o_done phases)
        int mg = 0;                                    // fused merges done (mrg_all / mrg_flag phases)
        load_q(h_start, 0);
        int4 ent_next = __ldg(&walk[e_start]);
        int h = h_start, e = e_start - 1;
        for (int j = 0; j < J; ++j) {
            if (++e == p.nwalk) {
                e = 0;
                ++h;
            }
            const bool seg_first = (j == 0) || (e == 0);
            const bool seg_last = (j == J - 1) || (e == p.nwalk - 1);
            if (seg_first) {
                m_run = -INFINITY;
                l_run = 0.f;
                // the next head's Q goes to the other buffer while this head runs;
                // that buffer's last reader (the previous head's QKs) has completed
                if (h < h_last) load_q(h + 1, (hs + 1) & 1);
                ++hs;
            }
            const int4 ent = ent_next;
            if (j + 1 < J) ent_next = __ldg(&walk[e + 1 == p.nwalk ? 0 : e + 1]);
            const int nvis = visible_prefix(p.rule, ent, qframe);
            const int b = (2 * j + t) % 3;
            const uint32_t t_s = tmem + lane_base + b * PAGE;

            if (!all_ok(wait_bar(s_full(b), ((2 * j + t) / 3) & 1, ctl))) break;
            fence_after();
            uint32_t r[PAGE];
            auto load_s = [&]() {
#pragma unroll
                for (int c = 0; c < PAGE / 32; ++c) tmem_ld32(t_s + 32 * c, r + 32 * c);
                tmem_wait_ld();
                if (nvis < PAGE) {
#pragma unroll
                    for (int c = 0; c < PAGE; ++c) r[c] = (c < nvis) ? r[c] : 0xff800000u;
                }
            };
            auto exps = [&](float msub) -> float {
                const uint64_t sl2v = f2(sl2, sl2);
                const uint64_t nmv = f2(-msub, -msub);
                uint64_t rs2[4] = {f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f)};
#pragma unroll
                for (int c = 0; c < PAGE; c += 2) {
                    const uint64_t x = ffma2(f2(__uint_as_float(r[c]), __uint_as_float(r[c + 1])), sl2v, nmv);
                    float x0, x1, p0, p1;
                    unf2(x, x0, x1);
                    p0 = ex2(x0);
                    p1 = ex2(x1);
                    rs2[(c >> 1) & 3] = fadd2(rs2[(c >> 1) & 3], f2(p0, p1));
                    r[c] = __float_as_uint(p0);
                    r[c + 1] = __float_as_uint(p1);
                }
                float s0, s1, s2, s3, s4, s5, s6, s7;
                unf2(rs2[0], s0, s1);
                unf2(rs2[1], s2, s3);
                unf2(rs2[2], s4, s5);
                unf2(rs2[3], s6, s7);
                return ((s0 + s1) + (s2 + s3)) + ((s4 + s5) + (s6 + s7));
            };
            load_s();

            float alpha = 1.f;
            bool resc = false;
            bool fast = m_run != -INFINITY;
            float rs = 0.f;
            if (fast) {
                rs = exps(m_run);
                fast = rs < 0x1p64f;
            }
            if (!__all_sync(0xffffffffu, fast)) {
                if (__any_sync(0xffffffffu, m_run != -INFINITY)) load_s();
                float acc[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) acc[i] = __uint_as_float(r[i]);
#pragma unroll
                for (int c = 16; c + 32 <= PAGE; c += 32)
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        acc[i] = fmax3(acc[i], __uint_as_float(r[c + i]), __uint_as_float(r[c + 16 + i]));
                if constexpr ((PAGE - 16) % 32 != 0) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) acc[i] = fmaxf(acc[i], __uint_as_float(r[PAGE - 16 + i]));
                }
                const float a0 = fmax3(acc[0], acc[1], acc[2]), a1 = fmax3(acc[3], acc[4], acc[5]);
                const float a2 = fmax3(acc[6], acc[7], acc[8]), a3 = fmax3(acc[9], acc[10], acc[11]);
                const float a4 = fmax3(acc[12], acc[13], acc[14]);
                const float mt = fmax3(fmax3(a0, a1, a2), fmax3(a3, a4, acc[15]), -INFINITY) * sl2;
                if (mt > m_run) {
                    if (m_run != -INFINITY) {
                        alpha = ex2(m_run - mt);
                        resc = true;
                    }
                    m_run = mt;
                }
                rs = exps(m_run == -INFINITY ? 0.f : m_run);
            }

            if (__any_sync(0xffffffffu, resc)) {
                // O_t holds PV_t up to page j-1 once that PV has completed
                // both tiles' PVs of page j-1 have completed once its K/V stage is released
                if (!all_ok(wait_bar(kv_empty((j - 1) % kStages), ((j - 1) / kStages) & 1, ctl))) break;
                fence_after();
                const uint64_t a2v = f2(alpha, alpha);
#pragma unroll 1
                for (int part = 0; part < 4; ++part) {
                    uint32_t o[16];
                    tmem_ld16(t_o + 16 * part, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int d = 0; d < 16; d += 2) {
                        float x0, x1;
                        unf2(fmul2(f2(__uint_as_float(o[d]), __uint_as_float(o[d + 1])), a2v), x0, x1);
                        o[d] = __float_as_uint(x0);
                        o[d + 1] = __float_as_uint(x1);
                    }
                    tmem_st16(t_o + 16 * part, o);
                }
            }

            // P (bf16) over the first PAGE/2 columns of the page's S buffer
#pragma unroll
            for (int c = 0; c < PAGE / 32; ++c) {
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    pk[i] = pack_bf16(__uint_as_float(r[32 * c + 2 * i]), __uint_as_float(r[32 * c + 2 * i + 1]));
                tmem_st16(t_s + 16 * c, pk);
            }
            l_run = l_run * alpha + rs;
            tmem_wait_st();
            fence_before();
            mbar_arrive(p_full(t, j & 1));

            if (seg_last) {
                // the head's last PV_t has completed -> O_t final for this head
                if (!all_ok(wait_bar(o_done(t), hd & 1, ctl))) break;
                ++hd;
                fence_after();
                uint32_t o[64];
                tmem_ld32(t_o, o);
                tmem_ld32(t_o + 32, o + 32);
                tmem_wait_ld();
                const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
                const float lse2 = l_run > 0.f ? m_run + __log2f(l_run) : -INFINITY;
                const int w_lo = (int)(((long long)h * p.nwalk) / p.seg);
                const int w_hi = (int)(((long long)(h + 1) * p.nwalk - 1) / p.seg);
                if (w_lo == w_hi) {
                    if (valid) {
                        uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) +
                                                              ((long long)row * p.H + h) * 64);
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            uint4 v;
                            v.x = pack_bf16(__uint_as_float(o[8 * i + 0]) * inv, __uint_as_float(o[8 * i + 1]) * inv);
                            v.y = pack_bf16(__uint_as_float(o[8 * i + 2]) * inv, __uint_as_float(o[8 * i + 3]) * inv);
                            v.z = pack_bf16(__uint_as_float(o[8 * i + 4]) * inv, __uint_as_float(o[8 * i + 5]) * inv);
                            v.w = pack_bf16(__uint_as_float(o[8 * i + 6]) * inv, __uint_as_float(o[8 * i + 7]) * inv);
                            dst[i] = v;
                        }
                        if (p.lse) p.lse[(long long)row * p.H + h] = lse2 * 0.69314718055994531f;
                    }
                } else {
                    // the head is split between workers: leave this worker's
                    // normalised partial and log2-sum-exp; the worker that
                    // finishes the head last combines all of them
                    const long long base = (long long)(qp * 2 + t) * (p.W + p.H - 1) + h;
                    if (valid) {
                        const long long slot = base + w;
                        float4* dst = reinterpret_cast<float4*>(p.ws_o + (slot * kRows + rl) * 64);
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            dst[i] = make_float4(__uint_as_float(o[4 * i + 0]) * inv, __uint_as_float(o[4 * i + 1]) * inv,
                                                 __uint_as_float(o[4 * i + 2]) * inv, __uint_as_float(o[4 * i + 3]) * inv);
                        p.ws_lse[slot * kRows + rl] = lse2;
                    }
                    __threadfence();
                    mbar_arrive(mrg_all(t));
                    if (!all_ok(wait_bar(mrg_all(t), mg & 1, ctl))) break;
                    if (rl == 0) {
                        // count the head's finished workers in this launch: the
                        // counter's high word is the launch epoch, the low word
                        // the count, so no reset between launches is needed
                        unsigned long long* cnt = p.merge_cnt + (long long)(qp * 2 + t) * p.H + h;
                        unsigned long long cur = *reinterpret_cast<volatile unsigned long long*>(cnt), nxt;
                        for (;;) {
                            nxt = ((unsigned long long)p.epoch << 32) |
                                  ((unsigned)(cur >> 32) == p.epoch ? (cur & 0xffffffffull) + 1 : 1ull);
                            const unsigned long long seen = atomicCAS(cnt, cur, nxt);
                            if (seen == cur) break;
                            cur = seen;
                        }
                        last_flag[t] = (int)(nxt & 0xffffffffull) == w_hi - w_lo + 1;
                        mbar_arrive(mrg_flag(t));
                    }
                    if (!all_ok(wait_bar(mrg_flag(t), mg & 1, ctl))) break;
                    ++mg;
                    if (last_flag[t] && valid) {
                        __threadfence();
                        float mx = -INFINITY;
                        for (int ww = w_lo; ww <= w_hi; ++ww)
                            mx = fmaxf(mx, __ldcg(p.ws_lse + (base + ww) * kRows + rl));
                        float acc[64];
#pragma unroll
                        for (int d = 0; d < 64; ++d) acc[d] = 0.f;
                        float den = 0.f;
                        for (int ww = w_lo; ww <= w_hi; ++ww) {
                            const float l2 = __ldcg(p.ws_lse + (base + ww) * kRows + rl);
                            if (l2 == -INFINITY) continue;
                            const float wt = ex2(l2 - mx);
                            den += wt;
                            const float4* src = reinterpret_cast<const float4*>(p.ws_o + ((base + ww) * kRows + rl) * 64);
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                const float4 v = __ldcg(src + i);
                                acc[4 * i + 0] = fmaf(wt, v.x, acc[4 * i + 0]);
                                acc[4 * i + 1] = fmaf(wt, v.y, acc[4 * i + 1]);
                                acc[4 * i + 2] = fmaf(wt, v.z, acc[4 * i + 2]);
                                acc[4 * i + 3] = fmaf(wt, v.w, acc[4 * i + 3]);
                            }
                        }
                        const float dinv = den > 0.f ? 1.f / den : 0.f;
                        uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) +
                                                              ((long long)row * p.H + h) * 64);
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            dst[i] = make_uint4(pack_bf16(acc[8 * i + 0] * dinv, acc[8 * i + 1] * dinv),
                                                pack_bf16(acc[8 * i + 2] * dinv, acc[8 * i + 3] * dinv),
                                                pack_bf16(acc[8 * i + 4] * dinv, acc[8 * i + 5] * dinv),
                                                pack_bf16(acc[8 * i + 6] * dinv, acc[8 * i + 7] * dinv));
                        if (p.lse)
                            p.lse[(long long)row * p.H + h] = (den > 0.f ? mx + __log2f(den) : -INFINITY) * 0.69314718055994531f;
                    }
                }
            }
        }
    }

    // ---------------------------------------------------------------- teardown
    fence_before();
    __syncthreads();
    if (warp == kWarpMMA) {
        fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(kTmemCols)
                     : "memory");
    }
}

// Self-test of the bounded wait: one thread waits on a barrier phase that
// nothing completes; the wait gives up after timeout_ns, raises the status
// word and the kernel returns.
__global__ void bounded_wait_selftest(int* status, unsigned long long timeout_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x != 0) return;
    abort_flag = 0;
    mbar_init(smem_u32(&bar), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    const Ctl ctl{&abort_flag, status};
    wait_bar(smem_u32(&bar), 0, ctl, true, timeout_ns);
}

template <int PAGE, bool BATCH>
cudaError_t launch_page(const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tkf,
                        const CUtensorMap& tvf, const AttendParams& p, cudaStream_t s) {
    const int smem = Layout<PAGE>::kSmemBytes;
    cudaError_t e = cudaFuncSetAttribute(attend_kernel<PAGE, BATCH>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dim3 grid((p.QT + 1) / 2, p.W);
    attend_kernel<PAGE, BATCH><<<grid, kThreads, smem, s>>>(tk, tv, tkf, tvf, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attend_sm100(const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tkf,
                                const CUtensorMap& tvf, const AttendParams& p, cudaStream_t s) {
    if (p.ppf > 0) {
        if (p.P == 128) return launch_page<128, true>(tk, tv, tkf, tvf, p, s);
        if (p.P == 64) return launch_page<64, true>(tk, tv, tkf, tvf, p, s);
        return cudaErrorInvalidValue;
    }
    if (p.P == 128) return launch_page<128, false>(tk, tv, tkf, tvf, p, s);
    if (p.P == 64) return launch_page<64, false>(tk, tv, tkf, tvf, p, s);
    return cudaErrorInvalidValue;
}

cudaError_t launch_bounded_wait_selftest(int* status, unsigned long long timeout_ns, cudaStream_t s) {
    bounded_wait_selftest<<<1, 32, 0, s>>>(status, timeout_ns);
    return cudaGetLastError();
}


}  // namespace gca
