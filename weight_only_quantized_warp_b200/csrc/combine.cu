// combine.cu -- router-weighted combine of the expert outputs.
//
// y[t] = rsf * sum_j w[t, j] * (o[inv[t, j]] + b2[e_j]) + shared[t], j in
// list order, fp32, rounded once to the output dtype (rsf: the
// routed_scaling_factor times the expert_output_scale; w = 1 when the
// weights scaled the expert inputs). The "MoE" page
// (clika_runtime.nn) combines the expert outputs under the router weights;
// "ClikaRT::nn::QMoEWoQ" forward() folds the optional shared_output into this
// routed combine (no separate add pass). Reading: the fc2 bias belongs to the
// expert output and is weighted with it. FC2 split-K partials are summed here
// in split order, so the result does not depend on scheduling.
#include "qmoe_internal.cuh"

namespace qmoe {
namespace {

constexpr int kCombineThreads = 256;
constexpr int kCombineChunk = kCombineThreads * 4;  // elements of one row per block

// One block per (token, 1024-element chunk of its row); each thread owns four
// consecutive elements. The token's k routes are read once per block; the
// loads of all k rows and splits are independent, so they are in flight
// together.
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(const CombineArgs a) {
    pdl_wait();  // every input comes from earlier kernels of the forward
    const float* __restrict__ o = a.o;
    const int nchunk = int((a.H + kCombineChunk - 1) / kCombineChunk);
    const int64_t nblk = a.T * nchunk;
    for (int64_t b = blockIdx.x; b < nblk; b += gridDim.x) {
        const int64_t t = b / nchunk;
        const int64_t m = (b - t * nchunk) * kCombineChunk + 4 * threadIdx.x;
        if (m >= a.H) continue;
        float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        for (int j = 0; j < a.k; ++j) {
            const int64_t pos = a.inv[t * a.k + j];
            const float w = a.weights_on_input ? 1.0f : a.topk_w[t * a.k + j];
            float v[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            for (int s = 0; s < a.splits; ++s) {
                const float4 p = __ldcs(reinterpret_cast<const float4*>(o + ((int64_t)s * a.R + pos) * a.H + m));
                v[0] += p.x;
                v[1] += p.y;
                v[2] += p.z;
                v[3] += p.w;
            }
            if (a.b2) {
                const int64_t e = a.topk_idx[t * a.k + j];
                const float4 bb = *reinterpret_cast<const float4*>(a.b2 + e * a.H + m);
                v[0] += bb.x;
                v[1] += bb.y;
                v[2] += bb.z;
                v[3] += bb.w;
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[q] = fmaf(w, v[q], acc[q]);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[q] *= a.rsf;
        if (a.act_bf16) {
            if (a.shared) {
                const uint2 sv = *reinterpret_cast<const uint2*>((const __nv_bfloat16*)a.shared + t * a.H + m);
                acc[0] += __uint_as_float(sv.x << 16);
                acc[1] += __uint_as_float(sv.x & 0xFFFF0000u);
                acc[2] += __uint_as_float(sv.y << 16);
                acc[3] += __uint_as_float(sv.y & 0xFFFF0000u);
            }
            __nv_bfloat162 lo = __floats2bfloat162_rn(acc[0], acc[1]);
            __nv_bfloat162 hi = __floats2bfloat162_rn(acc[2], acc[3]);
            uint2 out;
            out.x = *reinterpret_cast<uint32_t*>(&lo);
            out.y = *reinterpret_cast<uint32_t*>(&hi);
            *reinterpret_cast<uint2*>((__nv_bfloat16*)a.y + t * a.H + m) = out;
        } else {
            if (a.shared) {
                const float4 sv = *reinterpret_cast<const float4*>((const float*)a.shared + t * a.H + m);
                acc[0] += sv.x;
                acc[1] += sv.y;
                acc[2] += sv.z;
                acc[3] += sv.w;
            }
            *reinterpret_cast<float4*>((float*)a.y + t * a.H + m) = make_float4(acc[0], acc[1], acc[2], acc[3]);
        }
    }
}

}  // namespace

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t st) {
    if (a.T == 0) return cudaSuccess;
    int64_t blocks = a.T * ((a.H + kCombineChunk - 1) / kCombineChunk);
    if (blocks > 148 * 16) blocks = 148 * 16;
    return launch_kernel(combine_kernel, dim3(unsigned(blocks)), dim3(kCombineThreads), 0, st, a.pdl != 0, a);
}

}  // namespace qmoe
