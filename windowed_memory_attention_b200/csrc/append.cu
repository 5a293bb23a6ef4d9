// Append kernel: scatter one frame's token-major K and V into the page pools.
//
// Each step adds the new frame's M image tokens and S summary tokens to the
// cache (code walkthrough §2; paper digest §2.4).  Image token m of the frame
// goes to image page m / P, slot m % P; summary token s goes to the summary
// stream at index S*t + s.  Pools are [L][num_pages][H][P][D], so one
// (page, head) tile is a contiguous P x D block — the unit the attention
// kernel loads with one TMA box.
//
// The copy is HBM-bound: every 16-byte chunk is read once and written once.
// blockIdx.y selects (layer, tensor); the x dimension strides over 16-byte
// chunks in source order, so reads are fully coalesced and each group of
// D*elem/16 lanes writes whole 128-byte lines of one page row.
//
// Slots that no token fills (the tail of a frame's last image page, and the
// not-yet-used tail of a newly opened summary page) are zeroed, so a masked
// key never multiplies stale non-finite bytes in the PV product.
#include "gca_internal.h"

namespace gca {

namespace {

__device__ __forceinline__ int4 ld_stream(const int4* p) {
    int4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.s32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}

__global__ void __launch_bounds__(256) append_kernel(const AppendParams p) {
    const int lt = blockIdx.y;                 // layer-local index * 2 + tensor
    const int ll = lt >> 1;
    const int tensor = lt & 1;
    const int layer = p.layer0 + ll;
    const char* src = static_cast<const char*>(tensor ? p.v : p.k);
    char* pool = static_cast<char*>(tensor ? p.vpool : p.kpool);

    const int row_bytes = kHeadDim * p.elem_bytes;       // one token of one head
    const int cpr_shift = p.elem_bytes == 2 ? 3 : 4;     // 16-byte chunks per row: 8 or 16
    const unsigned cpr = 1u << cpr_shift;
    const long long tile_bytes = (long long)p.P * row_bytes;
    const long long layer_src = (long long)p.Lq * p.H * row_bytes;
    src += (long long)ll * layer_src;
    char* lpool = pool + (long long)layer * p.num_pages * p.H * tile_bytes;

    // 32-bit index arithmetic: one (layer, tensor) has at most Lq*H*16 chunks
    const unsigned H = (unsigned)p.H;
    const unsigned n_copy = (unsigned)p.Lq * H * cpr;
    // zero regions, per head: image tail slots and new summary page tail
    const unsigned img_tail = (p.M % p.P) ? (unsigned)(p.P - p.M % p.P) : 0u;
    unsigned sum_from = 0, sum_tail = 0;
    if (p.new_sum_seq >= 0) {
        sum_from = (unsigned)(p.S * (p.frame + 1) - p.new_sum_seq * p.P);   // first unused slot
        sum_tail = (unsigned)p.P - sum_from;
    }
    const unsigned n_zimg = H * img_tail * cpr;
    const unsigned n_zsum = H * sum_tail * cpr;
    const unsigned total = n_copy + n_zimg + n_zsum;

    // destination of chunk u (and whether it is a zero fill)
    auto dest = [&](unsigned u, bool& zero) -> char* {
        if (u < n_copy) {
            zero = false;
            const unsigned chunk = u & (cpr - 1);
            const unsigned th = u >> cpr_shift;
            const unsigned tau = th / H;
            const unsigned h = th - tau * H;
            int page, slot;
            if ((int)tau < p.S) {
                const int idx = p.S * p.frame + (int)tau;
                const int seq = idx / p.P;
                page = p.sum_page[seq - p.sum_seq0];
                slot = idx - seq * p.P;
            } else {
                const int m = (int)tau - p.S;
                const int seq = m / p.P;
                page = p.img_pages[seq];
                slot = m - seq * p.P;
            }
            return lpool + ((long long)page * p.H + h) * tile_bytes +
                   (long long)slot * row_bytes + chunk * 16;
        }
        zero = true;
        unsigned z = u - n_copy;
        int page;
        unsigned slot0, nslots;
        if (z < n_zimg) {
            page = p.img_pages[(p.M - 1) / p.P];
            slot0 = (unsigned)p.P - img_tail;
            nslots = img_tail;
        } else {
            z -= n_zimg;
            page = p.sum_page[p.new_sum_seq - p.sum_seq0];
            slot0 = sum_from;
            nslots = sum_tail;
        }
        const unsigned chunk = z & (cpr - 1);
        const unsigned ts = z >> cpr_shift;
        const unsigned h = ts / nslots;
        const unsigned sl = ts - h * nslots;
        return lpool + ((long long)page * p.H + h) * tile_bytes +
               (long long)(slot0 + sl) * row_bytes + chunk * 16;
    };

    // four independent chunks per thread per iteration: loads first, then stores
    constexpr int U = 4;
    const unsigned stride = gridDim.x * blockDim.x;
    for (unsigned base = blockIdx.x * blockDim.x + threadIdx.x; base < total; base += U * stride) {
        int4 val[U];
        char* dst[U];
        bool zero[U];
#pragma unroll
        for (int i = 0; i < U; ++i) {
            const unsigned u = base + i * stride;
            dst[i] = nullptr;
            if (u < total) {
                dst[i] = dest(u, zero[i]);
                val[i] = zero[i] ? make_int4(0, 0, 0, 0)
                                 : ld_stream(reinterpret_cast<const int4*>(src) + u);
            }
        }
#pragma unroll
        for (int i = 0; i < U; ++i)
            if (dst[i]) *reinterpret_cast<int4*>(dst[i]) = val[i];
    }
}

}  // namespace

cudaError_t launch_append(const AppendParams& p, cudaStream_t s) {
    const int sms = p.sms > 0 ? p.sms : 148;
    const long long per_lt = (long long)p.Lq * p.H * (kHeadDim * p.elem_bytes / 16);
    // about 4 chunks per thread per (layer, tensor), at most 8 blocks per SM overall
    long long want = (per_lt + 256 * 4 - 1) / (256 * 4);
    const long long cap = (8LL * sms + 2 * p.nlayers - 1) / (2 * p.nlayers);
    if (want > cap) want = cap;
    if (want < 1) want = 1;
    dim3 grid((unsigned)want, (unsigned)(2 * p.nlayers));
    append_kernel<<<grid, 256, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace gca
