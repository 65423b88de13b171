// combine.cu -- router-weighted combine of the expert outputs.
//
// y[t] = sum_j w[t, j] * (o[inv[t, j]] + b2[e_j]) + shared[t], j in list
// order, fp32, rounded once to the output dtype. The "MoE" page
// (clika_runtime.nn) combines the expert outputs under the router weights;
// "ClikaRT::nn::QMoEWoQ" forward() folds the optional shared_output into this
// routed combine (no separate add pass). Reading: the fc2 bias belongs to the
// expert output and is weighted with it. FC2 split-K partials are summed here
// in split order, so the result does not depend on scheduling.
#include "qmoe_internal.cuh"

namespace qmoe {
namespace {

__global__ void combine_kernel(const CombineArgs a) {
    const int64_t hq = a.H / 4;
    const int64_t total = a.T * hq;
    for (int64_t id = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; id < total;
         id += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = id / hq, m = (id % hq) * 4;
        float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        for (int j = 0; j < a.k; ++j) {
            const int64_t pos = a.inv[t * a.k + j];
            const float w = a.topk_w[t * a.k + j];
            float v[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            for (int s = 0; s < a.splits; ++s) {
                const float4 p = *reinterpret_cast<const float4*>(a.o + ((int64_t)s * a.R + pos) * a.H + m);
                v[0] += p.x;
                v[1] += p.y;
                v[2] += p.z;
                v[3] += p.w;
            }
            if (a.b2) {
                const int64_t e = a.topk_idx[t * a.k + j];
                const float4 b = *reinterpret_cast<const float4*>(a.b2 + e * a.H + m);
                v[0] += b.x;
                v[1] += b.y;
                v[2] += b.z;
                v[3] += b.w;
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[q] = fmaf(w, v[q], acc[q]);
        }
        if (a.act_bf16) {
            if (a.shared) {
                const __nv_bfloat16* s = (const __nv_bfloat16*)a.shared + t * a.H + m;
#pragma unroll
                for (int q = 0; q < 4; ++q) acc[q] += __bfloat162float(s[q]);
            }
            __nv_bfloat162 lo = __floats2bfloat162_rn(acc[0], acc[1]);
            __nv_bfloat162 hi = __floats2bfloat162_rn(acc[2], acc[3]);
            uint2 out;
            out.x = *reinterpret_cast<uint32_t*>(&lo);
            out.y = *reinterpret_cast<uint32_t*>(&hi);
            *reinterpret_cast<uint2*>((__nv_bfloat16*)a.y + t * a.H + m) = out;
        } else {
            if (a.shared) {
                const float4 s = *reinterpret_cast<const float4*>((const float*)a.shared + t * a.H + m);
                acc[0] += s.x;
                acc[1] += s.y;
                acc[2] += s.z;
                acc[3] += s.w;
            }
            *reinterpret_cast<float4*>((float*)a.y + t * a.H + m) =
                make_float4(acc[0], acc[1], acc[2], acc[3]);
        }
    }
}

}  // namespace

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t st) {
    const int threads = 256;
    int64_t blocks = (a.T * (a.H / 4) + threads - 1) / threads;
    if (blocks > 148 * 16) blocks = 148 * 16;
    if (blocks < 1) blocks = 1;
    combine_kernel<<<unsigned(blocks), threads, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace qmoe
