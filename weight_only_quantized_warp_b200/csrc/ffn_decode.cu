// ffn_decode.cu -- expert FFN layers that stream the packed weights.
//
// Each linear is y = x @ dequant(W).T + b ("QLinearWoQ" page, class summary)
// over the rows routed to one expert, with the weights decoded block by block
// inside the dot and never written out dense ("ClikaRT::nn::QMoEWoQ", class
// description). FC1 applies the gated activation of the QMoE page
// (activation_type, activation_alpha/beta, swiglu_limit) in its epilogue.
//
// Work split: one warp per 16-row weight tile, looping over the tile's
// k-groups (optionally a K-split of them) and over the expert's routed rows in
// passes of 8*NT tokens. The weight tile streams from HBM through a ring of
// D in-flight 16-byte loads per lane; activations (a few hundred KB at decode
// sizes) are read through L1.
//
// Fragments. For an m16n8k16 MMA, lane L holds A rows r0 = L/4 and r0 + 8 at
// k positions 2c, 2c+1, 2c+8, 2c+9 (c = L%4) and B column r0 at the same k
// positions. Because the dot product does not depend on the order of k, the
// packed layout assigns lane column c the 16 consecutive actual k
// [16c, 16c + 16) of each 64-wide group (int4; 8 of each 32-wide group for
// int8), spread over 4 (2) MMA k-steps. The lane's activations for a group are
// then one contiguous 32-byte (16-byte) run, and its weights one 16-byte load.
//
// Int-to-bf16 decode, derived from the IEEE-754 bf16 layout (1 sign, 8
// exponent, 7 mantissa bits): the word 0x4300 is 128.0 and its mantissa's unit
// in the last place is exactly 1, so OR-ing a 4-bit code q into the low
// mantissa bits gives exactly 128 + q, and subtracting 136.0 (0x4308) gives
// q - 8 exactly. Eight-bit codes do not fit a 7-bit mantissa, so they go
// through fp32: 0x4B000000 is 2^23 with unit 1, OR-ing the byte gives
// 2^23 + q, subtracting 2^23 + 128 gives q - 128 exactly, and the small
// integer converts to bf16 exactly.
//
// Scales. Per-column scales (block_size 0) and block scales spanning whole
// k-groups are applied in fp32 to the MMA partial of each block, so the MMA
// sees exact integer weights. Smaller blocks (16 and 32 for int4, 16 for
// int8) cover only part of a group's k-steps, so the scale is folded into the
// decoded bf16 weight instead (one rounding).
#include "qmoe_internal.cuh"

namespace qmoe {
namespace {

constexpr int kWarps = 8;

__device__ __forceinline__ uint4 ld_stream(const uint8_t* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint4 ld_act(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t bf2_sub(uint32_t a, uint32_t b) {
    __nv_bfloat162 r = __hsub2(*reinterpret_cast<__nv_bfloat162*>(&a),
                               *reinterpret_cast<__nv_bfloat162*>(&b));
    return *reinterpret_cast<uint32_t*>(&r);
}

__device__ __forceinline__ uint32_t bf2_mul(uint32_t a, uint32_t b) {
    __nv_bfloat162 r = __hmul2(*reinterpret_cast<__nv_bfloat162*>(&a),
                               *reinterpret_cast<__nv_bfloat162*>(&b));
    return *reinterpret_cast<uint32_t*>(&r);
}

__device__ __forceinline__ uint32_t pack_bf2(float lo, float hi) {
    __nv_bfloat162 r = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&r);
}

// 8 int4 codes -> 4 bf16x2 A registers holding q - 8 (register p takes nibble
// p in its low half and nibble p + 4 in its high half).
__device__ __forceinline__ void decode_int4(uint32_t w, uint32_t (&A)[4]) {
    constexpr uint32_t kMask = 0x000F000Fu, kMagic = 0x43004300u, kBias = 0x43084308u;
    A[0] = bf2_sub((w & kMask) | kMagic, kBias);
    A[1] = bf2_sub(((w >> 4) & kMask) | kMagic, kBias);
    A[2] = bf2_sub(((w >> 8) & kMask) | kMagic, kBias);
    A[3] = bf2_sub(((w >> 12) & kMask) | kMagic, kBias);
}

// byte m of w -> fp32 (q - 128), exactly
__device__ __forceinline__ float byte_centered(uint32_t w, int m) {
    return __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7440u | m)) - 8388736.0f;
}

// nibble p of w -> fp32 (q - 8), exactly
__device__ __forceinline__ float nibble_centered(uint32_t w, int p) {
    return __uint_as_float(0x4B000000u | ((w >> (4 * p)) & 0xFu)) - 8388616.0f;
}

__device__ __forceinline__ float load_scale(const void* S, int64_t i, bool f32) {
    if (f32) return ((const float*)S)[i];
    return __bfloat162float(((const __nv_bfloat16*)S)[i]);
}

// ------------------------------------------------------------- activations
__device__ __forceinline__ float sigmoidf_(float v) { return 1.0f / (1.0f + expf(-v)); }

__device__ __forceinline__ float act_plain(int t, float a) {
    switch (t) {
        case QMOE_ACT_RELU: return fmaxf(a, 0.0f);
        case QMOE_ACT_GELU: return 0.5f * a * (1.0f + erff(a * 0.70710678118654752f));
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
// (row r0+8, token 2c+1) of one 8-token tile starting at segment row p.
__device__ __forceinline__ void epilogue(const FfnArgs& a, int64_t rt, int r0, int c, int64_t seg0,
                                         int M, int p, const float (&v)[4], int split, bool out_bf16) {
    const int tA = p + 2 * c, tB = tA + 1;
    if (a.is_fc1) {
        if (a.gated) {
            const int64_t I = a.N / 2;
            const int64_t i = rt * 8 + r0;
            const float bg = a.bias ? a.bias[(int64_t)blockIdx.y * a.N + rt * 16 + r0] : 0.0f;
            const float bu = a.bias ? a.bias[(int64_t)blockIdx.y * a.N + rt * 16 + r0 + 8] : 0.0f;
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
            const float b0 = a.bias ? a.bias[(int64_t)blockIdx.y * a.N + m0] : 0.0f;
            const float b1 = a.bias ? a.bias[(int64_t)blockIdx.y * a.N + m1] : 0.0f;
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

// SMODE: 0 per-column scale after the K loop; 1 block scale after each
// block's MMAs; 2 block scale folded into the decoded weights.
template <int BITS, int SMODE, bool SF32, int NT>
__global__ void __launch_bounds__(kWarps * 32) ffn_decode_kernel(const FfnArgs a) {
    constexpr int KG = kgroup_of(BITS);
    constexpr int D = 8;  // weight loads in flight per lane
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int r0 = lane >> 2, c = lane & 3;
    const int e = blockIdx.y, split = blockIdx.z;
    const int64_t nrt = a.N / kTileRows;
    const int64_t rt = (int64_t)blockIdx.x * kWarps + warp;
    if (rt >= nrt) return;
    const int64_t seg0 = a.offsets[e];
    const int M = a.offsets[e + 1] - int(seg0);
    if (M <= 0) return;
    const int64_t ngr = a.K / KG;
    const int64_t nsb = a.block_size > 0 ? a.K / a.block_size : 1;
    const int64_t gpb = (SMODE == 1) ? a.block_size / KG : 1;
    int64_t g_lo, g_hi;
    split_range(ngr, a.splits, split, gpb, g_lo, g_hi);

    const uint8_t* wtile = a.W + ((int64_t)e * nrt + rt) * ngr * kUnitBytes + lane * 16;
    const int64_t sbase = ((int64_t)e * nrt + rt) * nsb * 16 + 2 * r0;  // scale of row r0; +1 = r0+8
    const __nv_bfloat16* act = (const __nv_bfloat16*)a.act;

    float s0 = 1.0f, s1 = 1.0f;  // per-column scales
    if (SMODE == 0) {
        s0 = load_scale(a.S, sbase, SF32);
        s1 = load_scale(a.S, sbase + 1, SF32);
    }

    for (int p0 = 0; p0 < M; p0 += 8 * NT) {
        const __nv_bfloat16* xrow[NT];
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            const int tok = min(p0 + 8 * n + r0, M - 1);
            const int64_t row = a.rowmap ? a.rowmap[seg0 + tok] : seg0 + tok;
            xrow[n] = act + row * a.K + (KG / 4) * c;
        }
        float acc[NT][4], blk[NT][4];
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[n][q] = blk[n][q] = 0.0f;

        uint4 wr[D];
#pragma unroll
        for (int i = 0; i < D; ++i)
            if (g_lo + i < g_hi) wr[i] = ld_stream(wtile + (g_lo + i) * kUnitBytes);

        for (int64_t g = g_lo; g < g_hi; g += D) {
#pragma unroll
            for (int i = 0; i < D; ++i) {
                const int64_t gi = g + i;
                if (gi < g_hi) {
                    const uint4 w = wr[i];
                    if (gi + D < g_hi) wr[i] = ld_stream(wtile + (gi + D) * kUnitBytes);
                    // activations of this group: 16 (int4) or 8 (int8) bf16 per token tile
                    uint4 xa[NT][2];
#pragma unroll
                    for (int n = 0; n < NT; ++n) {
                        xa[n][0] = ld_act(xrow[n] + gi * KG);
                        if (BITS == 4) xa[n][1] = ld_act(xrow[n] + gi * KG + 8);
                    }
                    // scales of this lane's block
                    float sa = 1.0f, sb = 1.0f;
                    if (SMODE == 1) {
                        const int64_t b = gi * KG / a.block_size;
                        sa = load_scale(a.S, sbase + b * 16, SF32);
                        sb = load_scale(a.S, sbase + b * 16 + 1, SF32);
                    } else if (SMODE == 2) {
                        const int64_t b = (gi * KG + (KG / 4) * c) / a.block_size;
                        sa = load_scale(a.S, sbase + b * 16, SF32);
                        sb = load_scale(a.S, sbase + b * 16 + 1, SF32);
                    }
                    const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
                    constexpr int KSTEPS = BITS == 4 ? 4 : 2;
#pragma unroll
                    for (int j = 0; j < KSTEPS; ++j) {
                        uint32_t A[4];
                        if (BITS == 4) {
                            if (SMODE == 2 && SF32) {
                                const uint32_t x = wv[j];
#pragma unroll
                                for (int q = 0; q < 4; ++q) {
                                    const float sc = (q & 1) ? sb : sa;
                                    A[q] = pack_bf2(nibble_centered(x, q) * sc,
                                                    nibble_centered(x, q + 4) * sc);
                                }
                            } else {
                                decode_int4(wv[j], A);
                                if (SMODE == 2) {
                                    const __nv_bfloat162 pa = __float2bfloat162_rn(sa);
                                    const __nv_bfloat162 pb = __float2bfloat162_rn(sb);
                                    const uint32_t ua = *reinterpret_cast<const uint32_t*>(&pa);
                                    const uint32_t ub = *reinterpret_cast<const uint32_t*>(&pb);
                                    A[0] = bf2_mul(A[0], ua);
                                    A[1] = bf2_mul(A[1], ub);
                                    A[2] = bf2_mul(A[2], ua);
                                    A[3] = bf2_mul(A[3], ub);
                                }
                            }
                        } else {
                            const uint32_t lo = wv[2 * j], hi = wv[2 * j + 1];
                            float f[8];
#pragma unroll
                            for (int m = 0; m < 4; ++m) {
                                f[m] = byte_centered(lo, m);
                                f[4 + m] = byte_centered(hi, m);
                            }
                            if (SMODE == 2) {
                                if (SF32) {
#pragma unroll
                                    for (int m = 0; m < 8; ++m) f[m] *= ((m >> 1) & 1) ? sb : sa;
                                } else {
                                    const float ra = __bfloat162float(__float2bfloat16_rn(sa));
                                    const float rb = __bfloat162float(__float2bfloat16_rn(sb));
#pragma unroll
                                    for (int m = 0; m < 8; ++m) f[m] *= ((m >> 1) & 1) ? rb : ra;
                                }
                            }
#pragma unroll
                            for (int q = 0; q < 4; ++q) A[q] = pack_bf2(f[2 * q], f[2 * q + 1]);
                        }
#pragma unroll
                        for (int n = 0; n < NT; ++n) {
                            const uint32_t* xw = reinterpret_cast<const uint32_t*>(&xa[n][0]);
                            // kstep j uses activation words 2j, 2j+1 of the lane's run
                            if (SMODE == 1)
                                mma_bf16(blk[n], A, xw[2 * j], xw[2 * j + 1]);
                            else
                                mma_bf16(acc[n], A, xw[2 * j], xw[2 * j + 1]);
                        }
                    }
                    if (SMODE == 1 && (((gi + 1) % gpb) == 0 || gi + 1 == g_hi)) {
#pragma unroll
                        for (int n = 0; n < NT; ++n) {
                            acc[n][0] = fmaf(sa, blk[n][0], acc[n][0]);
                            acc[n][1] = fmaf(sa, blk[n][1], acc[n][1]);
                            acc[n][2] = fmaf(sb, blk[n][2], acc[n][2]);
                            acc[n][3] = fmaf(sb, blk[n][3], acc[n][3]);
                            blk[n][0] = blk[n][1] = blk[n][2] = blk[n][3] = 0.0f;
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            float v[4] = {acc[n][0], acc[n][1], acc[n][2], acc[n][3]};
            if (SMODE == 0) {
                v[0] *= s0;
                v[1] *= s0;
                v[2] *= s1;
                v[3] *= s1;
            }
            epilogue(a, rt, r0, c, seg0, M, p0 + 8 * n, v, split, true);
        }
    }
}

// fp32 activations: the same tiling with FFMA (fp32 accumulation of exact
// integer codes times fp32 activations, scaled per lane block).
template <int BITS>
__global__ void __launch_bounds__(kWarps * 32) ffn_simt_kernel(const FfnArgs a) {
    constexpr int KG = kgroup_of(BITS);
    constexpr int KL = KG / 4;  // actual k per lane per group
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int r0 = lane >> 2, c = lane & 3;
    const int e = blockIdx.y, split = blockIdx.z;
    const int64_t nrt = a.N / kTileRows;
    const int64_t rt = (int64_t)blockIdx.x * kWarps + warp;
    if (rt >= nrt) return;
    const int64_t seg0 = a.offsets[e];
    const int M = a.offsets[e + 1] - int(seg0);
    if (M <= 0) return;
    const int64_t ngr = a.K / KG;
    const int64_t nsb = a.block_size > 0 ? a.K / a.block_size : 1;
    int64_t g_lo, g_hi;
    split_range(ngr, a.splits, split, 1, g_lo, g_hi);
    const uint8_t* wtile = a.W + ((int64_t)e * nrt + rt) * ngr * kUnitBytes + lane * 16;
    const int64_t sbase = ((int64_t)e * nrt + rt) * nsb * 16 + 2 * r0;
    const float* act = (const float*)a.act;
    const bool sf32 = !a.scale_bf16;

    for (int p0 = 0; p0 < M; p0 += 8) {
        // this lane reduces all 8 tokens of the tile over its k sub-range
        const float* xrow[8];
#pragma unroll
        for (int n = 0; n < 8; ++n) {
            const int tok = min(p0 + n, M - 1);
            const int64_t row = a.rowmap ? a.rowmap[seg0 + tok] : seg0 + tok;
            xrow[n] = act + row * a.K + KL * c;
        }
        float acc[8][2];
#pragma unroll
        for (int n = 0; n < 8; ++n) acc[n][0] = acc[n][1] = 0.0f;
        for (int64_t g = g_lo; g < g_hi; ++g) {
            const uint4 w = *reinterpret_cast<const uint4*>(wtile + g * kUnitBytes);
            const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
            // decode the lane's 2 x KL codes into (row, actual k) order
            float q[2][KL];
            if (BITS == 4) {
#pragma unroll
                for (int j = 0; j < 4; ++j)
#pragma unroll
                    for (int p = 0; p < 8; ++p)
                        q[p & 1][4 * j + 2 * ((p >> 1) & 1) + (p >> 2)] = nibble_centered(wv[j], p);
            } else {
#pragma unroll
                for (int j = 0; j < 2; ++j)
#pragma unroll
                    for (int m = 0; m < 8; ++m) {
                        const int qq = m >> 1;
                        q[qq & 1][4 * j + 2 * (qq >> 1) + (m & 1)] =
                            byte_centered(wv[2 * j + (m >> 2)], m & 3);
                    }
            }
            const int64_t b = a.block_size > 0 ? (g * KG + KL * c) / a.block_size : 0;
            const float sa = load_scale(a.S, sbase + b * 16, sf32);
            const float sb = load_scale(a.S, sbase + b * 16 + 1, sf32);
#pragma unroll
            for (int n = 0; n < 8; ++n) {
                float pa = 0.0f, pb = 0.0f;
#pragma unroll
                for (int v4 = 0; v4 < KL / 4; ++v4) {
                    const float4 xv = *reinterpret_cast<const float4*>(xrow[n] + g * KG + 4 * v4);
                    const float xs[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        pa = fmaf(q[0][4 * v4 + u], xs[u], pa);
                        pb = fmaf(q[1][4 * v4 + u], xs[u], pb);
                    }
                }
                acc[n][0] = fmaf(sa, pa, acc[n][0]);
                acc[n][1] = fmaf(sb, pb, acc[n][1]);
            }
        }
        // reduce over the 4 lanes of a row pair (lane bits 0-1)
#pragma unroll
        for (int n = 0; n < 8; ++n)
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                acc[n][r] += __shfl_xor_sync(0xffffffffu, acc[n][r], 1);
                acc[n][r] += __shfl_xor_sync(0xffffffffu, acc[n][r], 2);
            }
        // lane c takes tokens 2c, 2c+1, as in the MMA C fragment
        float v[4];
#pragma unroll
        for (int n = 0; n < 8; ++n) {
            if (n == 2 * c) {
                v[0] = acc[n][0];
                v[2] = acc[n][1];
            }
            if (n == 2 * c + 1) {
                v[1] = acc[n][0];
                v[3] = acc[n][1];
            }
        }
        epilogue(a, rt, r0, c, seg0, M, p0, v, split, false);
    }
}

template <int BITS, int SMODE, bool SF32>
cudaError_t launch_nt(const FfnArgs& a, dim3 grid, cudaStream_t st) {
    switch (a.nt) {
        case 1: ffn_decode_kernel<BITS, SMODE, SF32, 1><<<grid, kWarps * 32, 0, st>>>(a); break;
        case 2: ffn_decode_kernel<BITS, SMODE, SF32, 2><<<grid, kWarps * 32, 0, st>>>(a); break;
        default: ffn_decode_kernel<BITS, SMODE, SF32, 4><<<grid, kWarps * 32, 0, st>>>(a); break;
    }
    return cudaGetLastError();
}

template <int BITS, int SMODE>
cudaError_t launch_sf(const FfnArgs& a, dim3 grid, cudaStream_t st) {
    return a.scale_bf16 ? launch_nt<BITS, SMODE, false>(a, grid, st)
                        : launch_nt<BITS, SMODE, true>(a, grid, st);
}

}  // namespace

int scale_mode(int bits, int block_size) {
    if (block_size == 0) return 0;
    return block_size >= kgroup_of(bits) ? 1 : 2;
}

cudaError_t launch_ffn_decode(const FfnArgs& a, cudaStream_t st) {
    const int64_t nrt = a.N / kTileRows;
    dim3 grid(unsigned((nrt + kWarps - 1) / kWarps), unsigned(a.E), unsigned(a.splits));
    const int sm = scale_mode(a.bits, a.block_size);
    if (a.bits == 4) {
        if (sm == 0) return launch_sf<4, 0>(a, grid, st);
        if (sm == 1) return launch_sf<4, 1>(a, grid, st);
        return launch_sf<4, 2>(a, grid, st);
    }
    if (sm == 0) return launch_sf<8, 0>(a, grid, st);
    if (sm == 1) return launch_sf<8, 1>(a, grid, st);
    return launch_sf<8, 2>(a, grid, st);
}

cudaError_t launch_ffn_simt(const FfnArgs& a, cudaStream_t st) {
    const int64_t nrt = a.N / kTileRows;
    dim3 grid(unsigned((nrt + kWarps - 1) / kWarps), unsigned(a.E), unsigned(a.splits));
    if (a.bits == 4)
        ffn_simt_kernel<4><<<grid, kWarps * 32, 0, st>>>(a);
    else
        ffn_simt_kernel<8><<<grid, kWarps * 32, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace qmoe
