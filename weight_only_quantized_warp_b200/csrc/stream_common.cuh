// stream_common.cuh -- pieces shared by the weight-streaming mma.sync
// kernels (the bf16 decode kernels and the int8 block-tier kernels): the
// streaming weight load, the cp.async staging helpers, the K-split range, the
// per-tile scale pair and the FC1/FC2 epilogue with the gated activations of
// the QMoE page (activation_type, activation_alpha/beta, swiglu_limit).
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

#include "qmoe_internal.cuh"

namespace qmoe {
namespace {

__device__ __forceinline__ uint4 ld_stream(const uint8_t* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// ------------------------------------------------------------- activations
__device__ __forceinline__ float sigmoidf_(float v) { return 1.0f / (1.0f + expf(-v)); }

__device__ __forceinline__ float act_plain(int t, float a) {
    switch (t) {
        case QMOE_ACT_RELU: return fmaxf(a, 0.0f);
        case QMOE_ACT_GELU: return 0.5f * a * (1.0f + erff(a * 0.70710678118654752f));
        case kActGeluTanh: return 0.5f * a * (1.0f + tanhf(0.79788456080286536f * (a + 0.044715f * a * a * a)));
        case QMOE_ACT_SILU: return a * sigmoidf_(a);
        default: return a;
    }
}

// alpha and limit arrive already resolved (alpha 0 -> 1, no limit -> +inf).
__device__ __forceinline__ float act_gated(int t, float g, float u, float alpha, float beta,
                                           float limit) {
    if (t == QMOE_ACT_SWIGLU) {
        g = fminf(g, limit);
        u = fminf(fmaxf(u, -limit), limit);
        return (u + beta) * g * sigmoidf_(alpha * g);
    }
    return act_plain(t, g) * u;
}

__device__ __forceinline__ void store_act(void* p, int64_t i, float v, bool bf16) {
    if (bf16)
        ((__nv_bfloat16*)p)[i] = __float2bfloat16_rn(v);
    else
        ((float*)p)[i] = v;
}

// Shared epilogue. v[0..3] are the MMA C-fragment values of lane (r0, c):
// (row r0, token 2c), (row r0, token 2c+1), (row r0+8, token 2c),
// (row r0+8, token 2c+1) of one 8-token tile starting at segment row p of
// expert e.
__device__ __forceinline__ void epilogue(const FfnArgs& a, int e, int64_t rt, int r0, int c, int64_t seg0,
                                         int M, int p, const float (&v)[4], int split, bool out_bf16) {
    const int tA = p + 2 * c, tB = tA + 1;
    if (a.is_fc1) {
        if (a.gated) {
            const int64_t I = a.N / 2;
            const int64_t i = rt * 8 + r0;
            const float bg = a.bias ? a.bias[(int64_t)e * a.N + rt * 16 + r0] : 0.0f;
            const float bu = a.bias ? a.bias[(int64_t)e * a.N + rt * 16 + r0 + 8] : 0.0f;
            if (tA < M)
                store_act(a.out, (seg0 + tA) * I + i,
                          act_gated(a.act_type, v[0] + bg, v[2] + bu, a.alpha, a.beta, a.limit),
                          out_bf16);
            if (tB < M)
                store_act(a.out, (seg0 + tB) * I + i,
                          act_gated(a.act_type, v[1] + bg, v[3] + bu, a.alpha, a.beta, a.limit),
                          out_bf16);
        } else {
            const int64_t I = a.N;
            const int64_t m0 = rt * 16 + r0, m1 = m0 + 8;
            const float b0 = a.bias ? a.bias[(int64_t)e * a.N + m0] : 0.0f;
            const float b1 = a.bias ? a.bias[(int64_t)e * a.N + m1] : 0.0f;
            if (tA < M) {
                store_act(a.out, (seg0 + tA) * I + m0, act_plain(a.act_type, v[0] + b0), out_bf16);
                store_act(a.out, (seg0 + tA) * I + m1, act_plain(a.act_type, v[2] + b1), out_bf16);
            }
            if (tB < M) {
                store_act(a.out, (seg0 + tB) * I + m0, act_plain(a.act_type, v[1] + b0), out_bf16);
                store_act(a.out, (seg0 + tB) * I + m1, act_plain(a.act_type, v[3] + b1), out_bf16);
            }
        }
    } else {
        float* o = (float*)a.out + (int64_t)split * a.R * a.N;
        const int64_t m0 = rt * 16 + r0, m1 = m0 + 8;
        if (tA < M) {
            o[(seg0 + tA) * a.N + m0] = v[0];
            o[(seg0 + tA) * a.N + m1] = v[2];
        }
        if (tB < M) {
            o[(seg0 + tB) * a.N + m0] = v[1];
            o[(seg0 + tB) * a.N + m1] = v[3];
        }
    }
}

// k-group range of one split; splits cut on block boundaries when the scale
// is applied per block after the MMA.
__device__ __forceinline__ void split_range(int64_t ngr, int splits, int split, int64_t gpb,
                                            int64_t& lo, int64_t& hi) {
    const int64_t nblk = (ngr + gpb - 1) / gpb;
    const int64_t per = (nblk + splits - 1) / splits;
    lo = min(ngr, split * per * gpb);
    hi = min(ngr, (split + 1) * per * gpb);
}

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
    const uint32_t d = uint32_t(__cvta_generic_to_shared(smem_dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gsrc) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.wait_all;" ::: "memory");
}

// Raw scale pair (rows r0, r0 + 8) of one row tile and block: two bf16 in one
// word, or two fp32.
template <bool F32>
struct ScaleRaw;
template <>
struct ScaleRaw<false> {
    uint32_t v;
    __device__ __forceinline__ static ScaleRaw load(const void* S, int idx) {
        return {*reinterpret_cast<const uint32_t*>((const __nv_bfloat16*)S + idx)};
    }
    __device__ __forceinline__ void get(float& sa, float& sb) const {
        sa = __uint_as_float(v << 16);
        sb = __uint_as_float(v & 0xFFFF0000u);
    }
};
template <>
struct ScaleRaw<true> {
    float2 v;
    __device__ __forceinline__ static ScaleRaw load(const void* S, int idx) {
        return {*reinterpret_cast<const float2*>((const float*)S + idx)};
    }
    __device__ __forceinline__ void get(float& sa, float& sb) const {
        sa = v.x;
        sb = v.y;
    }
};

}  // namespace
}  // namespace qmoe
