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
//
// With the 3D rotary encoding on, K is rotated as it is stored: each dim pair
// (2i, 2i+1) of token u turns by the angle of its axis (frame time for pairs
// 0..11, patch row and column for 12..31), in fp32, and is rounded back to
// the cache dtype (see RopeTables).
#include <cuda_bf16.h>

#include "gca_internal.h"

namespace gca {

namespace {

__device__ __forceinline__ int4 ld_stream(const int4* p) {
    int4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.s32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}

#ifndef GCA_APPEND_U
#define GCA_APPEND_U 4
#endif
#ifndef GCA_APPEND_BLOCKS_PER_SM
#define GCA_APPEND_BLOCKS_PER_SM 8
#endif

// HSHIFT = log2(H) when H is a power of two (shifts instead of divisions), else -1;
// ROPE: K is rotated by the 3D rotary encoding (a separate instantiation keeps
// the plain copy's register count, and so its occupancy, unchanged)
template <int HSHIFT, bool ROPE>
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
    const int p_shift = p.P == 128 ? 7 : 6;              // P is 64 or 128
    const unsigned img_tail = (p.M % p.P) ? (unsigned)(p.P - p.M % p.P) : 0u;
    unsigned sum_from = 0, sum_tail = 0;
    if (p.new_sum_seq >= 0) {
        sum_from = (unsigned)(p.S * (p.frame + 1) - p.new_sum_seq * p.P);   // first unused slot
        sum_tail = (unsigned)p.P - sum_from;
    }
    const unsigned n_zimg = H * img_tail * cpr;
    const unsigned n_zsum = H * sum_tail * cpr;
    const unsigned total = n_copy + n_zimg + n_zsum;

    // destination of chunk u (and whether it is a zero fill); tok / chunk: the
    // chunk's token in the frame and its 16-byte index within the head's row
    auto dest = [&](unsigned u, bool& zero, unsigned& tok, unsigned& chunk) -> char* {
        if (u < n_copy) {
            zero = false;
            chunk = u & (cpr - 1);
            const unsigned th = u >> cpr_shift;
            const unsigned tau = HSHIFT >= 0 ? th >> HSHIFT : th / H;
            tok = tau;
            const unsigned h = HSHIFT >= 0 ? th & ((1u << (HSHIFT & 31)) - 1u) : th - tau * H;
            int page, slot;
            if ((int)tau < p.S) {
                const int idx = p.S * p.frame + (int)tau;
                const int seq = idx >> p_shift;
                page = p.sum_page[seq - p.sum_seq0];
                slot = idx & (p.P - 1);
            } else {
                const int m = (int)tau - p.S;
                page = p.img_pages[m >> p_shift];
                slot = m & (p.P - 1);
            }
            return lpool + ((long long)page * p.H + h) * tile_bytes +
                   (long long)slot * row_bytes + chunk * 16;
        }
        zero = true;
        tok = 0;
        chunk = 0;
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
        const unsigned zc = z & (cpr - 1);
        const unsigned ts = z >> cpr_shift;
        const unsigned h = ts / nslots;
        const unsigned sl = ts - h * nslots;
        return lpool + ((long long)page * p.H + h) * tile_bytes +
               (long long)(slot0 + sl) * row_bytes + zc * 16;
    };
    // K with the 3D rotary encoding: each 16-byte chunk holds whole dim pairs
    const bool rotate = ROPE && tensor == 0;
    auto rope_chunk = [&](int4& v, unsigned tok, unsigned chunk) {
        if (p.elem_bytes == 2) {
            uint32_t w[4] = {(uint32_t)v.x, (uint32_t)v.y, (uint32_t)v.z, (uint32_t)v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                __nv_bfloat162 b2 = *reinterpret_cast<__nv_bfloat162*>(&w[j]);
                float a = __low2float(b2), b = __high2float(b2);
                rope_rotate(a, b, rope_cs(p.rope, p.rope_t, (int)tok, (int)chunk * 4 + j));
                b2 = __floats2bfloat162_rn(a, b);
                w[j] = *reinterpret_cast<uint32_t*>(&b2);
            }
            v = make_int4((int)w[0], (int)w[1], (int)w[2], (int)w[3]);
        } else {
            float f[4] = {__int_as_float(v.x), __int_as_float(v.y), __int_as_float(v.z), __int_as_float(v.w)};
            rope_rotate(f[0], f[1], rope_cs(p.rope, p.rope_t, (int)tok, (int)chunk * 2));
            rope_rotate(f[2], f[3], rope_cs(p.rope, p.rope_t, (int)tok, (int)chunk * 2 + 1));
            v = make_int4(__float_as_int(f[0]), __float_as_int(f[1]), __float_as_int(f[2]), __float_as_int(f[3]));
        }
    };

    // four independent chunks per thread per iteration: loads first, then stores
    constexpr int U = GCA_APPEND_U;
    const unsigned stride = gridDim.x * blockDim.x;
    for (unsigned base = blockIdx.x * blockDim.x + threadIdx.x; base < total; base += U * stride) {
        int4 val[U];
        char* dst[U];
        bool zero[U];
        unsigned tok[U], chunk[U];
#pragma unroll
        for (int i = 0; i < U; ++i) {
            const unsigned u = base + i * stride;
            dst[i] = nullptr;
            if (u < total) {
                dst[i] = dest(u, zero[i], tok[i], chunk[i]);
                val[i] = zero[i] ? make_int4(0, 0, 0, 0)
                                 : ld_stream(reinterpret_cast<const int4*>(src) + u);
            }
        }
        if constexpr (ROPE) {
            if (rotate) {
#pragma unroll
                for (int i = 0; i < U; ++i)
                    if (dst[i] && !zero[i]) rope_chunk(val[i], tok[i], chunk[i]);
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
    // about U chunks per thread per (layer, tensor), a bounded number of blocks per SM overall
    constexpr int U = GCA_APPEND_U;
    long long want = (per_lt + 256 * U - 1) / (256 * U);
    const long long cap = ((long long)GCA_APPEND_BLOCKS_PER_SM * sms + 2 * p.nlayers - 1) / (2 * p.nlayers);
    if (want > cap) want = cap;
    if (want < 1) want = 1;
    dim3 grid((unsigned)want, (unsigned)(2 * p.nlayers));
    const int hs = (p.H & (p.H - 1)) == 0 ? __builtin_ctz((unsigned)p.H) : -1;
    if (p.rope.t) {
        if (hs == 4) append_kernel<4, true><<<grid, 256, 0, s>>>(p);
        else append_kernel<-1, true><<<grid, 256, 0, s>>>(p);
        return cudaGetLastError();
    }
    switch (hs) {
        case 0: append_kernel<0, false><<<grid, 256, 0, s>>>(p); break;
        case 1: append_kernel<1, false><<<grid, 256, 0, s>>>(p); break;
        case 2: append_kernel<2, false><<<grid, 256, 0, s>>>(p); break;
        case 3: append_kernel<3, false><<<grid, 256, 0, s>>>(p); break;
        case 4: append_kernel<4, false><<<grid, 256, 0, s>>>(p); break;
        case 5: append_kernel<5, false><<<grid, 256, 0, s>>>(p); break;
        default: append_kernel<-1, false><<<grid, 256, 0, s>>>(p); break;
    }
    return cudaGetLastError();
}

}  // namespace gca
