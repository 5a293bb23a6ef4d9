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
// leave normalised partials plus their log-sum-exp for the merge kernel.
//
// Per CTA (384 threads, one CTA per SM):
//   warps 0-3 / 4-7  softmax of tile 0 / tile 1: thread t owns query row t of
//              its tile (TMEM lane t); loads Q into TMEM, reads S rows from
//              TMEM, online softmax in the log2 domain, writes P (bf16) back
//              over the S columns, final normalisation;
//   warp 8     TMA producer: one (page, head) K tile and V tile per stage,
//              128-byte swizzled boxes of P x 64 bf16, 4 stages;
//   warp 9     MMA issuer (one thread) and TMEM owner (warps 10-11 idle).
//              Per page j it issues
//                S0 = Q0 K_j^T,  O1 += P1(j-1) V_{j-1},  S1 = Q1 K_j^T,
//                O0 += P0(j) V_j
//              so each softmax group overlaps the other group's two MMAs
//              (A = Q or P from TMEM, B = K K-major / V MN-major from smem).
// TMEM columns: S0, S1 (P aliased into their first P/2 columns), O0, O1, Q0,
// Q1 — 448 of 512 for 128-token pages.  tcgen05 operations issued by one
// thread execute in order, so S_t(j+1) is written only after PV_t(j) has read
// P_t(j), and the commit after QK_t(j+1) also covers PV_t(j).
//
// Softmax: a page is exponentiated against the row's running max without
// computing the page max first.  Since relative precision does not depend on
// scale, values up to 2^64 are as good as values up to 1; a row whose page
// sum reaches 2^64 (or overflows) takes the exact path instead: page max, O
// rescaled by 2^(m_old - m_new), exponentials recomputed.  The first page of
// every head always takes the exact path.  Scores are scaled and shifted with
// packed f32x2 FMAs; two of every sixteen column pairs get 2^x from a
// degree-3 minimax polynomial on the FMA pipe (exp2_poly_fit.py), the rest
// from the MUFU unit (ex2.approx).
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
#ifndef GCA_ATTEND_STAGES
#define GCA_ATTEND_STAGES 4
#endif
#ifndef GCA_POLY_PAIRS
#define GCA_POLY_PAIRS 2
#endif
constexpr int kStages = GCA_ATTEND_STAGES;
constexpr int kRows = 128;
constexpr uint32_t kTmemCols = 512;
constexpr unsigned long long kTimeoutNs = 2000000000ull;
constexpr int kPolyPairs = GCA_POLY_PAIRS;  // of each 16 column pairs, this many use the FMA-pipe 2^x

// 2^f on [-1/2, 1/2], minimax relative error 7.5e-5 (exp2_poly_fit.py)
constexpr float kExpC0 = 0x1.fff692p-1f;
constexpr float kExpC1 = 0x1.62f31ap-1f;
constexpr float kExpC2 = 0x1.f0de1ap-3f;
constexpr float kExpC3 = 0x1.c3f76p-5f;

template <int PAGE>
struct Layout {
    static constexpr int kTileBytes = PAGE * 128;          // PAGE x 64 bf16
    static constexpr int kStageBytes = 2 * kTileBytes;     // K then V
    static constexpr int kColS = 0;                        // + tile * PAGE (P in the first PAGE/2)
    static constexpr int kColO = 2 * PAGE;                 // + tile * 64
    static constexpr int kColQ = 2 * PAGE + 128;           // + tile * 32
    static_assert(kColQ + 64 <= (int)kTmemCols, "TMEM budget");
    static constexpr int kNumBars = 2 * kStages + 9;
    static constexpr int kSmemBytes = kStages * kStageBytes + kNumBars * 8 + 16 + 1024;
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
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        GCA_W8(0), GCA_W8(8), GCA_W8(16), GCA_W8(24)
        : "memory");
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

// 2^x for two values on the FMA pipe: x = j + f, j = rne(x) through the
// 1.5*2^23 shifter, p(f) by Horner, then j added to the exponent field.
// x is clamped to >= -125 so the exponent never underflows into the sign;
// an input below -125 (a masked key's -inf among them) gives exactly 0.
__device__ __forceinline__ void exp2_poly2(float x0, float x1, float& y0, float& y1) {
    const bool z0 = x0 < -125.f, z1 = x1 < -125.f;
    x0 = fmaxf(x0, -125.f);
    x1 = fmaxf(x1, -125.f);
    const uint64_t x = f2(x0, x1);
    const uint64_t t = fadd2(x, f2(12582912.f, 12582912.f));
    const uint64_t j = fadd2(t, f2(-12582912.f, -12582912.f));
    const uint64_t f = ffma2(j, f2(-1.f, -1.f), x);
    uint64_t p = ffma2(f2(kExpC3, kExpC3), f, f2(kExpC2, kExpC2));
    p = ffma2(p, f, f2(kExpC1, kExpC1));
    p = ffma2(p, f, f2(kExpC0, kExpC0));
    float t0, t1, p0, p1;
    unf2(t, t0, t1);
    unf2(p, p0, p1);
    y0 = __uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23));
    y1 = __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23));
    y0 = z0 ? 0.f : y0;
    y1 = z1 ? 0.f : y1;
}

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------
template <int PAGE>
__global__ void __launch_bounds__(kThreads, 1)
attend_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
              const AttendParams p) {
    using L = Layout<PAGE>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(smem);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * L::kStageBytes);
    const uint32_t bar0 = smem_u32(bars);
    auto kv_full = [&](int s) { return bar0 + 8u * s; };
    auto kv_empty = [&](int s) { return bar0 + 8u * (kStages + s); };
    auto s_full = [&](int t) { return bar0 + 8u * (2 * kStages + t); };
    auto p_full = [&](int t) { return bar0 + 8u * (2 * kStages + 2 + t); };
    auto pv_done = [&](int t) { return bar0 + 8u * (2 * kStages + 4 + t); };
    auto q_ready = [&](int t) { return bar0 + 8u * (2 * kStages + 6 + t); };
    const uint32_t drain = bar0 + 8u * (2 * kStages + 8);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + L::kNumBars);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const Ctl ctl{abort_flag, p.status};

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int qp = blockIdx.x;                 // pair of 128-row query tiles
    const int w = blockIdx.y;                  // worker (segment of the page stream)
    const long long total = (long long)p.H * p.nwalk;
    const long long g0 = (long long)w * p.seg;
    const long long g1 = (g0 + p.seg < total) ? g0 + p.seg : total;
    const int J = (int)(g1 - g0);
    // (head, entry) of the first page; every role then steps them incrementally
    const int h_start = (int)(g0 / p.nwalk);
    const int e_start = (int)(g0 - (long long)h_start * p.nwalk);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(kv_full(s), 1);
            mbar_init(kv_empty(s), 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(s_full(t), 1);
            mbar_init(p_full(t), kRows);
            mbar_init(pv_done(t), 1);
            mbar_init(q_ready(t), kRows);
        }
        mbar_init(drain, 1);
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
                const int page = __ldg(&p.walk[e].x);
                if (page < 0 || page >= p.num_pages) {
                    *abort_flag = 1;
                    *(volatile int*)p.status = kStatusBadPage;
                    ok = false;
                    break;
                }
                const int y = ((p.layer * p.num_pages + page) * p.H + h) * PAGE;
                const uint32_t dst = sbase + st * L::kStageBytes;
                mbar_expect_tx(kv_full(st), 2 * L::kTileBytes);
                tma_load_2d(dst, &tmK, 0, y, kv_full(st));
                tma_load_2d(dst + L::kTileBytes, &tmV, 0, y, kv_full(st));
                ++issued;
                if (++e == p.nwalk) {
                    e = 0;
                    ++h;
                }
            }
            if (!ok) {
                // let every load already issued land before the CTA exits
                const int from = issued > kStages ? issued - kStages : 0;
                for (int j = from; j < issued; ++j)
                    wait_bar(kv_full(j % kStages), (j / kStages) & 1, ctl, false);
            }
        }
        __syncwarp();
    } else if (warp == kWarpMMA) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t kIdescQK = idesc_bf16(kRows, PAGE, false);
            constexpr uint32_t kIdescPV = idesc_bf16(kRows, 64, true);
            // descriptors of stage 0; stage s and step kk add constants to the
            // start-address field (16-byte units): K steps 32 bytes, V steps 2 KB
            const uint64_t kdesc0 = desc_sw128(sbase, 16, 1024);
            const uint64_t vdesc0 = desc_sw128(sbase + L::kTileBytes, L::kTileBytes, 1024);
            constexpr uint64_t kStageStep = L::kStageBytes >> 4;
            // descriptor halves: only the low word (start address) varies
            const uint32_t kd_lo0 = (uint32_t)kdesc0, kd_hi = (uint32_t)(kdesc0 >> 32);
            const uint32_t vd_lo0 = (uint32_t)vdesc0, vd_hi = (uint32_t)(vdesc0 >> 32);
            auto qk = [&](int t, int st) {
                const uint64_t kd = kdesc0 + st * kStageStep;
                const uint32_t kd_lo = kd_lo0 + st * (uint32_t)kStageStep;
                const uint32_t scol = tmem + L::kColS + t * PAGE;
                const uint32_t qcol = tmem + L::kColQ + t * 32;
                mma_ts(scol, qcol, kd, kIdescQK, 0u);
#pragma unroll
                for (int kk = 1; kk < 4; ++kk)   // 16 head dims per step
                    mma_ts_acc(scol, qcol + kk * 8, kd_lo + 2 * kk, kd_hi, kIdescQK);
                mma_commit(s_full(t));
            };
            // pv_done is only needed at the end of a head: the commit after the
            // next QK_t covers PV_t for the softmax
            auto pv = [&](int t, int j, int st, bool first, bool last) -> bool {
                if (!wait_bar(p_full(t), j & 1, ctl)) return false;
                fence_after();
                const uint64_t vd = vdesc0 + st * kStageStep;
                const uint32_t vd_lo = vd_lo0 + st * (uint32_t)kStageStep;
                const uint32_t ocol = tmem + L::kColO + t * 64;
                const uint32_t pcol = tmem + L::kColS + t * PAGE;
                mma_ts(ocol, pcol, vd, kIdescPV, first ? 0u : 1u);
#pragma unroll
                for (int kk = 1; kk < PAGE / 16; ++kk)   // 16 keys per step
                    mma_ts_acc(ocol, pcol + kk * 8, vd_lo + 128 * kk, vd_hi, kIdescPV);
                if (last) mma_commit(pv_done(t));
                if (t == 1) mma_commit(kv_empty(st));
                return true;
            };
            bool ok = true;
            int sidx = 0;
            int e = e_start;
            bool prev_first = false, prev_last = false;
            int st = 0, prev_st = 0;
            for (int j = 0; j < J; ++j) {
                const bool seg_first = (j == 0) || (e == 0);
                const bool seg_last = (j == J - 1) || (e == p.nwalk - 1);
                if (seg_first && !wait_bar(q_ready(0), sidx & 1, ctl)) { ok = false; break; }
                if (!wait_bar(kv_full(st), (j / kStages) & 1, ctl)) { ok = false; break; }
                fence_after();
                qk(0, st);
                if (j > 0 && !pv(1, j - 1, prev_st, prev_first, prev_last)) { ok = false; break; }
                if (seg_first) {
                    if (!wait_bar(q_ready(1), sidx & 1, ctl)) { ok = false; break; }
                    ++sidx;
                    fence_after();
                }
                qk(1, st);
                if (!pv(0, j, st, seg_first, seg_last)) { ok = false; break; }
                prev_first = seg_first;
                prev_last = seg_last;
                prev_st = st;
                st = (st + 1 == kStages) ? 0 : st + 1;
                if (++e == p.nwalk) e = 0;
            }
            if (ok) pv(1, J - 1, prev_st, prev_first, prev_last);
            // drain: every MMA issued above completes before TMEM is released
            mma_commit(drain);
            wait_bar(drain, 0, ctl, false);
        }
        __syncwarp();
      }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
        // ------------------------------------------------------------ softmax
        const int t = warp >> 2;                       // query tile of this warp group
        const int quarter = warp & 3;
        const int rl = quarter * 32 + lane;            // row in the tile, TMEM lane
        const int row = (qp * 2 + t) * kRows + rl;
        const bool valid = row < p.R;
        const int qframe = p.first_query_frame + (valid ? row / p.Lq : 0);
        const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
        const uint32_t t_s = tmem + lane_base + L::kColS + t * PAGE;
        const uint32_t t_o = tmem + lane_base + L::kColO + t * 64;
        const uint32_t t_q = tmem + lane_base + L::kColQ + t * 32;
        const float sl2 = p.scale_log2;
        const __nv_bfloat16* qg = static_cast<const __nv_bfloat16*>(p.q);

        auto load_q = [&](int h) {
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
                    // 3D rotary encoding at the row's (frame, token) position:
                    // each 32-bit word holds dim pair i in fp32, rounded back to bf16
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
            tmem_st32(t_q, r);
            tmem_wait_st();
            fence_before();
            mbar_arrive(q_ready(t));
        };
        auto all_ok = [&](bool ok) { return __all_sync(0xffffffffu, ok); };

        float m_run = -INFINITY, l_run = 0.f;
        int segs_done = 0;                             // pv_done(t) phases consumed
        load_q(h_start);
        // walk entries are read one page ahead, off the critical path
        int4 ent_next = __ldg(&p.walk[e_start]);
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
            }
            const int4 ent = ent_next;
            if (j + 1 < J) ent_next = __ldg(&p.walk[e + 1 == p.nwalk ? 0 : e + 1]);
            const int nvis = visible_prefix(p.rule, ent, qframe);

            // S_t(j) is complete, and so is PV_t(j-1) (one commit covers both)
            if (!all_ok(wait_bar(s_full(t), j & 1, ctl))) break;
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
            // r <- 2^(s * scale_log2 - msub) in place; returns the row sum
            auto exps = [&](float msub) -> float {
                const uint64_t sl2v = f2(sl2, sl2);
                const uint64_t nmv = f2(-msub, -msub);
                uint64_t rs2[4] = {f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f)};
#pragma unroll
                for (int c = 0; c < PAGE; c += 2) {
                    const uint64_t x = ffma2(f2(__uint_as_float(r[c]), __uint_as_float(r[c + 1])), sl2v, nmv);
                    float x0, x1, p0, p1;
                    unf2(x, x0, x1);
                    if (((c >> 1) & 15) < kPolyPairs) {
                        exp2_poly2(x0, x1, p0, p1);
                    } else {
                        p0 = ex2(x0);
                        p1 = ex2(x1);
                    }
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

            // Fast path: exponentiate against the running max without looking
            // for this page's max.  Values up to 2^64 are exact enough (relative
            // precision does not depend on scale) and far from overflow; a row
            // whose page sum reaches 2^64 (or inf / NaN) takes the exact path.
            float alpha = 1.f;
            bool resc = false;
            bool fast = m_run != -INFINITY;
            float rs = 0.f;
            if (fast) {
                rs = exps(m_run);
                fast = rs < 0x1p64f;
            }
            if (!__all_sync(0xffffffffu, fast)) {
                // r was overwritten by a fast attempt in some lanes; the reload is
                // warp-collective, so every lane of the warp takes it
                if (__any_sync(0xffffffffu, m_run != -INFINITY)) load_s();
                // exact row max: 16 independent three-input max chains, then a tree
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
                // PV_t(j-1) has completed (covered by the s_full commit)
                const uint64_t a2v = f2(alpha, alpha);
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t o[32];
                    tmem_ld32(t_o + 32 * half, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int d = 0; d < 32; d += 2) {
                        float x0, x1;
                        unf2(fmul2(f2(__uint_as_float(o[d]), __uint_as_float(o[d + 1])), a2v), x0, x1);
                        o[d] = __float_as_uint(x0);
                        o[d + 1] = __float_as_uint(x1);
                    }
                    tmem_st32(t_o + 32 * half, o);
                }
            }

            // P (bf16) written over the S columns
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
            mbar_arrive(p_full(t));

            if (seg_last) {
                if (!all_ok(wait_bar(pv_done(t), segs_done & 1, ctl))) break;
                ++segs_done;
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
                } else if (valid) {
                    const long long slot = (long long)(qp * 2 + t) * (p.W + p.H - 1) + w + h;
                    float4* dst = reinterpret_cast<float4*>(p.ws_o + (slot * kRows + rl) * 64);
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        dst[i] = make_float4(__uint_as_float(o[4 * i + 0]) * inv, __uint_as_float(o[4 * i + 1]) * inv,
                                             __uint_as_float(o[4 * i + 2]) * inv, __uint_as_float(o[4 * i + 3]) * inv);
                    p.ws_lse[slot * kRows + rl] = lse2;
                }
                if (j < J - 1) load_q(h + 1);
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

// Combine the partials of heads that were split between workers.
__global__ void __launch_bounds__(128) merge_kernel(const AttendParams p) {
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (long long)p.R * p.H) return;
    const int row = (int)(idx / p.H);
    const int h = (int)(idx - (long long)row * p.H);
    const int w_lo = (int)(((long long)h * p.nwalk) / p.seg);
    const int w_hi = (int)(((long long)(h + 1) * p.nwalk - 1) / p.seg);
    if (w_lo == w_hi) return;
    const int qt = row / kRows, rl = row % kRows;
    const long long base = (long long)qt * (p.W + p.H - 1) + h;
    float mx = -INFINITY;
    for (int w = w_lo; w <= w_hi; ++w) mx = fmaxf(mx, p.ws_lse[(base + w) * kRows + rl]);
    float acc[64];
#pragma unroll
    for (int d = 0; d < 64; ++d) acc[d] = 0.f;
    float den = 0.f;
    for (int w = w_lo; w <= w_hi; ++w) {
        const float l2 = p.ws_lse[(base + w) * kRows + rl];
        if (l2 == -INFINITY) continue;
        const float wt = exp2f(l2 - mx);
        den += wt;
        const float4* src = reinterpret_cast<const float4*>(p.ws_o + ((base + w) * kRows + rl) * 64);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float4 v = src[i];
            acc[4 * i + 0] += wt * v.x;
            acc[4 * i + 1] += wt * v.y;
            acc[4 * i + 2] += wt * v.z;
            acc[4 * i + 3] += wt * v.w;
        }
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + ((long long)row * p.H + h) * 64);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        uint4 v;
        v.x = pack_bf16(acc[8 * i + 0] * inv, acc[8 * i + 1] * inv);
        v.y = pack_bf16(acc[8 * i + 2] * inv, acc[8 * i + 3] * inv);
        v.z = pack_bf16(acc[8 * i + 4] * inv, acc[8 * i + 5] * inv);
        v.w = pack_bf16(acc[8 * i + 6] * inv, acc[8 * i + 7] * inv);
        dst[i] = v;
    }
    if (p.lse) p.lse[(long long)row * p.H + h] = (mx + log2f(den)) * 0.69314718055994531f;
}

template <int PAGE>
cudaError_t launch_page(const CUtensorMap& tk, const CUtensorMap& tv, const AttendParams& p,
                        cudaStream_t s) {
    const int smem = Layout<PAGE>::kSmemBytes;
    cudaError_t e = cudaFuncSetAttribute(attend_kernel<PAGE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dim3 grid((p.QT + 1) / 2, p.W);
    attend_kernel<PAGE><<<grid, kThreads, smem, s>>>(tk, tv, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attend_sm100(const CUtensorMap& tk, const CUtensorMap& tv,
                                const AttendParams& p, cudaStream_t s) {
    if (p.P == 128) return launch_page<128>(tk, tv, p, s);
    if (p.P == 64) return launch_page<64>(tk, tv, p, s);
    return cudaErrorInvalidValue;
}

cudaError_t launch_bounded_wait_selftest(int* status, unsigned long long timeout_ns, cudaStream_t s) {
    bounded_wait_selftest<<<1, 32, 0, s>>>(status, timeout_ns);
    return cudaGetLastError();
}

cudaError_t launch_merge(const AttendParams& p, cudaStream_t s) {
    const long long n = (long long)p.R * p.H;
    merge_kernel<<<(unsigned)((n + 127) / 128), 128, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace gca
