// GCA attention in fp32 on the CUDA cores (the fp32 dtype of the cache).
//
// Same visibility rule and walk list as the tcgen05 path (paper digest §2.5):
// row r of the query block attends to the visible prefix of every walk-list
// page.  One thread owns one (row, head); the block stages one page's K and V
// tile (P x 64 fp32 each) in shared memory and every thread streams through it
// with an fp32 online softmax (natural exponent).  tf32 tensor-core products
// would lose the fp32 stream's precision, so this dtype stays on FMA units.
#include "gca_internal.h"

namespace gca {

namespace {

constexpr int kRowsPerBlock = 128;

__global__ void __launch_bounds__(kRowsPerBlock)
attend_f32_kernel(const AttendParams p, const float* __restrict__ kpool,
                  const float* __restrict__ vpool) {
    extern __shared__ float4 sm4[];
    float* ks = reinterpret_cast<float*>(sm4);
    float* vs = ks + p.P * kHeadDim;
    const int h = blockIdx.y;
    const int row = blockIdx.x * kRowsPerBlock + threadIdx.x;
    const bool valid = row < p.R;
    const int qframe = p.first_query_frame + (valid ? row / p.Lq : 0);

    float q[kHeadDim], acc[kHeadDim];
    const float* qg = static_cast<const float*>(p.q) + ((long long)(valid ? row : 0) * p.H + h) * kHeadDim;
#pragma unroll
    for (int d = 0; d < kHeadDim; ++d) {
        q[d] = valid ? qg[d] : 0.f;
        acc[d] = 0.f;
    }
    if (p.rope.t) {      // 3D rotary encoding of the query at its frame's position
        const int u = valid ? row % p.Lq : 0;
#pragma unroll
        for (int i = 0; i < kHeadDim / 2; ++i) rope_rotate(q[2 * i], q[2 * i + 1], rope_cs(p.rope, qframe, u, i));
    }
#pragma unroll
    for (int d = 0; d < kHeadDim; ++d) q[d] *= p.scale;
    float m = -INFINITY, l = 0.f;
    const long long tile = (long long)p.P * kHeadDim;
    for (int e = 0; e < p.nwalk; ++e) {
        const int4 ent = p.walk[e];
        const int page = ent.x;
        if (page < 0 || page >= p.num_pages) {
            if (threadIdx.x == 0) *(volatile int*)p.status = kStatusBadPage;
            break;   // uniform across the block: every thread reads the same entry
        }
        const long long off = (((long long)p.layer * p.num_pages + page) * p.H + h) * tile;
        const float4* kg = reinterpret_cast<const float4*>(kpool + off);
        const float4* vg = reinterpret_cast<const float4*>(vpool + off);
        for (int i = threadIdx.x; i < p.P * kHeadDim / 4; i += kRowsPerBlock) {
            sm4[i] = kg[i];
            sm4[p.P * kHeadDim / 4 + i] = vg[i];
        }
        __syncthreads();
        const int nv = visible_prefix(p.rule, ent, qframe);
        for (int u = 0; u < nv; ++u) {
            const float* ku = ks + u * kHeadDim;
            float s = 0.f;
#pragma unroll
            for (int d = 0; d < kHeadDim; ++d) s = fmaf(q[d], ku[d], s);
            const float* vu = vs + u * kHeadDim;
            if (s > m) {
                const float c = expf(m - s);     // 0 on the first key
                l *= c;
#pragma unroll
                for (int d = 0; d < kHeadDim; ++d) acc[d] *= c;
                m = s;
            }
            const float pr = expf(s - m);
            l += pr;
#pragma unroll
            for (int d = 0; d < kHeadDim; ++d) acc[d] = fmaf(pr, vu[d], acc[d]);
        }
        __syncthreads();
    }
    if (!valid) return;
    const float inv = l > 0.f ? 1.f / l : 0.f;
    float* o = static_cast<float*>(p.out) + ((long long)row * p.H + h) * kHeadDim;
#pragma unroll
    for (int d = 0; d < kHeadDim; ++d) o[d] = acc[d] * inv;
    if (p.lse) p.lse[(long long)row * p.H + h] = l > 0.f ? m + logf(l) : -INFINITY;
}

}  // namespace

cudaError_t launch_attend_f32(const AttendParams& p, const void* kpool, const void* vpool,
                              cudaStream_t s) {
    const int smem = 2 * p.P * kHeadDim * (int)sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(attend_f32_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dim3 grid((p.R + kRowsPerBlock - 1) / kRowsPerBlock, p.H);
    attend_f32_kernel<<<grid, kRowsPerBlock, smem, s>>>(p, static_cast<const float*>(kpool),
                                                        static_cast<const float*>(vpool));
    return cudaGetLastError();
}

}  // namespace gca
