// ffn_decode.cu -- expert FFN layers that stream the packed weights.
//
// Each linear is y = x @ dequant(W).T + b ("QLinearWoQ" page, class summary)
// over the rows routed to one expert, with the weights decoded block by block
// inside the dot and never written out dense ("ClikaRT::nn::QMoEWoQ", class
// description). FC1 applies the gated activation of the QMoE page
// (activation_type, activation_alpha/beta, swiglu_limit) in its epilogue.
//
// Work split: one CTA per (128-row weight block, expert, K-split), one warp
// per 16-row tile of the block, looping over the tile's k-groups and over the
// expert's routed rows in passes of 8*NT tokens. The weight tile streams from
// HBM through a ring of D in-flight 16-byte loads per lane (scales ride along
// in a parallel ring); the pass's activation rows are staged once per CTA in
// shared memory with cp.async.
//
// Fragments. For an m16n8k16 MMA, lane L holds A rows r0 = L/4 and r0 + 8 at
// k positions 2c, 2c+1, 2c+8, 2c+9 (c = L%4) and B column r0 at the same k
// positions. The packed layout maps those positions of k-step j to the actual
// k values 16j + 4c + {0, 1} and 16j + 4c + {2, 3} (the dot product does not
// depend on the order of k), so the lane's activations for one k-step are one
// 8-byte run and its weights for a whole k-group one 16-byte load.
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
#include <algorithm>

#include "qmoe_internal.cuh"
#include "fp4_decode.cuh"
#include "stream_common.cuh"

namespace qmoe {
namespace {

constexpr int kWarps = 8;

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D = A*B (accumulator input zero): starts a fresh partial without zeroing registers
__device__ __forceinline__ void mma_bf16_zero(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                              uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%10,%10,%10,%10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.0f));
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

// Bytes of one staged activation row for a k range of kr elements: bf16
// values plus 32 bytes of padding, so the 8-byte reads of 4 rows x 4 lanes
// that one phase of a warp's load serves land in distinct shared-memory banks.
__host__ __device__ constexpr int64_t staged_row_bytes(int64_t kr) { return kr * 2 + 32; }

// Zero-point folding (int4, scale after the MMA). With A = 128 + q (the code
// OR-ed into bf16 128.0, no subtraction), sum_k (q - 8) x_k equals
// sum_k A_k x_k - 136 * sum_k x_k. The activation sums per scale chunk and
// token are computed once per CTA pass from the staged rows, so the weight
// decode is 7 bit operations per 8 codes. The products A_k x_k are exact in
// fp32; the subtraction cancels a term about 17x the result, which costs a few
// fp32 ulp of that larger term.
constexpr float kFoldOffset = 136.0f;  // 128 (bf16 magic) + 8 (zero point)
constexpr int kRing = 8;               // weight loads in flight per lane

// SMODE: 0 per-column scale after the K loop; 1 block scale applied to the MMA
// partial every P k-groups (P = min(groups per block, kRing), so a block may
// be applied in several chunks with the same scale); 2 block scale folded
// into the decoded weights (P = 1).
//
// One CTA = 8 warps = the 8 row tiles of one 128-row block of one expert, for
// one K-split. The CTA stages the activation rows of its current 8*NT tokens
// (its K range only) in shared memory with cp.async, while every warp already
// has its first kRing weight loads in flight. The k-group loop has a steady
// part (loads always in range, no guards), one guarded drain round and a
// tail; all shared-memory, weight and scale addresses advance by constants.
// Resident CTAs per SM the kernel is built for: three for one 8-token tile
// (80 registers hold it), two for two or four tiles (whose accumulators and
// activation fragments would spill at 80).
template <int BITS, int SMODE, bool SF32, int NT, int P>
__global__ void __launch_bounds__(kWarps * 32, NT == 1 ? 3 : 2) ffn_decode_kernel(const FfnArgs a) {
    constexpr int KG = kgroup_of(BITS);
    constexpr int D = kRing;
    static_assert(D % P == 0, "scale chunk must divide the ring");
    constexpr bool FOLD = (BITS == 4 && SMODE != 2);
    constexpr int GS = kTilesPerBlock * kUnitBytes;  // group stride, 4 KB
    constexpr int ROWS = 8 * NT;
    constexpr int KSTEPS = BITS == 4 ? 4 : 2;
    constexpr int LG_KG = BITS == 4 ? 6 : 5;
    extern __shared__ __align__(16) uint8_t xs[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int r0 = lane >> 2, c = lane & 3;
    const int e = blockIdx.y, split = blockIdx.z;
    const int64_t rb = blockIdx.x;
    const int64_t nrt = a.N / kTileRows;
    const int64_t nrb = padded_rows(a.N) / kBlockRows;
    const int64_t rt = rb * kTilesPerBlock + warp;
    const bool active = rt < nrt;
    const int64_t ngr = a.K / KG;
    const int64_t nsb = a.block_size > 0 ? a.K / a.block_size : 1;
    const int lg_bs = a.block_size > 0 ? __ffs(a.block_size) - 1 : 0;
    const int lg_gpb = SMODE == 1 ? lg_bs - LG_KG : 0;
    int64_t g_lo, g_hi;
    split_range(ngr, a.splits, split, SMODE == 1 ? (int64_t(1) << lg_gpb) : 1, g_lo, g_hi);
    const int ng = int(g_hi - g_lo);
    const int kr = ng * KG;
    const int rs = int(staged_row_bytes(kr));
    const int chunks = kr / 8;  // 16-byte chunks per staged row
    // activation sums for the zero-point fold: [chunk of P groups][row]
    // (SMODE 1) or [row] (SMODE 0)
    float* cs = reinterpret_cast<float*>(xs + ROWS * rs);
    const int nch = FOLD ? (SMODE == 1 ? ng / P : 1) : 0;

    const uint8_t* wp =
        a.W + (((int64_t)e * nrb + rb) * ngr * kTilesPerBlock + warp) * kUnitBytes + lane * 16 +
        g_lo * GS;
    // scale pairs of this tile and lane (rows r0, r0 + 8): base pointer, then
    // a 32-bit index per chunk
    const int64_t sb0 = (((int64_t)e * nrb + rb) * nsb * kTilesPerBlock + warp) * 16 + 2 * r0;
    const void* sbase = SF32 ? (const void*)((const float*)a.S + sb0)
                             : (const void*)((const __nv_bfloat16*)a.S + sb0);
    // SMODE 1: scale index of absolute group ga; SMODE 2: of k-step j of ga
    auto sidx = [&](int ga) -> int { return (ga >> lg_gpb) * 128; };
    auto sidx_step = [&](int ga, int j) -> int { return ((ga * KG + 16 * j + 4 * c) >> lg_bs) * 128; };
    const __nv_bfloat16* act = (const __nv_bfloat16*)a.act;

    float s0 = 1.0f, s1 = 1.0f;  // per-column scales
    if (SMODE == 0 && active) ScaleRaw<SF32>::load(sbase, 0).get(s0, s1);

    // the first D k-groups of a pass (and their scales) in flight
    uint4 wr[D];
    ScaleRaw<SF32> sr[D / P];
    auto fill = [&]() {
        if (active) {
#pragma unroll
            for (int i = 0; i < D; ++i) {
                if (i < ng) {
                    wr[i] = ld_stream(wp + i * GS);
                    if (SMODE == 1 && i % P == 0) sr[i / P] = ScaleRaw<SF32>::load(sbase, sidx(int(g_lo) + i));
                }
            }
        }
    };
    // The weights depend on nothing the forward computes, so the first pass's
    // loads go out before the wait on the kernel before this one (routing or
    // FC1) when launched as its programmatic dependent; the segment offsets,
    // the row map and the activations are read only after it.
    fill();
    pdl_trigger();
    pdl_wait();
    const int64_t seg0 = a.offsets[e];
    const int M = a.offsets[e + 1] - int(seg0);
    if (M <= 0) return;  // uniform over the CTA

    for (int p0 = 0; p0 < M; p0 += ROWS) {
        if (p0 > 0) fill();
        // stage the activation rows of tokens p0 .. p0 + ROWS - 1 (clamped):
        // one warp per row, lanes over its 16-byte chunks
        for (int row = warp; row < ROWS; row += kWarps) {
            const int tok = min(p0 + row, M - 1);
            const int64_t srow = a.rowmap ? a.rowmap[seg0 + tok] : seg0 + tok;
            const __nv_bfloat16* src = act + srow * a.K + g_lo * KG;
            uint8_t* dst = xs + row * rs;
            for (int ch = lane; ch < chunks; ch += 32) cp_async16(dst + ch * 16, src + ch * 8);
        }
        cp_async_wait_all();
        __syncthreads();
        if (FOLD) {
            if (SMODE == 1) {
                // one thread per (chunk, row): fp32 sum in k order
                constexpr int CK = P * KG;  // k per chunk
                for (int i = tid; i < nch * ROWS; i += blockDim.x) {
                    const int b = i / ROWS, row = i - b * ROWS;
                    const uint4* src = reinterpret_cast<const uint4*>(xs + row * rs + b * CK * 2);
                    float sum = 0.0f;
#pragma unroll 4
                    for (int q = 0; q < CK / 8; ++q) {
                        const uint4 v = src[q];
                        const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                        for (int h = 0; h < 4; ++h) {
                            sum += __uint_as_float(u[h] << 16);
                            sum += __uint_as_float(u[h] & 0xFFFF0000u);
                        }
                    }
                    cs[i] = sum;
                }
            } else {
                // one warp per row: strided partial sums, then a fixed shuffle tree
                for (int row = warp; row < ROWS; row += kWarps) {
                    const uint4* src = reinterpret_cast<const uint4*>(xs + row * rs);
                    float sum = 0.0f;
                    for (int q = lane; q < chunks; q += 32) {
                        const uint4 v = src[q];
                        const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                        for (int h = 0; h < 4; ++h) {
                            sum += __uint_as_float(u[h] << 16);
                            sum += __uint_as_float(u[h] & 0xFFFF0000u);
                        }
                    }
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
                    if (lane == 0) cs[row] = sum;
                }
            }
            __syncthreads();
        }

        float acc[NT][4], blk[NT][4];
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[n][q] = blk[n][q] = 0.0f;

        // one k-group: decode the lane's 16 bytes, 4 (int4) or 2 (int8) MMA
        // k-steps per token tile. xg is this lane's activation run of the group.
        // first: this group opens a scale chunk (SMODE 1), so its first k-step
        // writes the chunk partial instead of adding to it
        auto group = [&](const uint4 w, const uint8_t* xg, const ScaleRaw<SF32> sc, int ga, bool first) {
            uint2 xa[NT][KSTEPS];  // per k-step: activation pairs at 16j+4c, 16j+4c+2
#pragma unroll
            for (int n = 0; n < NT; ++n)
#pragma unroll
                for (int j = 0; j < KSTEPS; ++j)
                    xa[n][j] = *reinterpret_cast<const uint2*>(xg + n * 8 * rs + j * 32);
            const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int j = 0; j < KSTEPS; ++j) {
                uint32_t A[4];
                float sa = 1.0f, sb = 1.0f;  // SMODE 2: scales of this k-step's block
                if (SMODE == 2) ScaleRaw<SF32>::load(sbase, sidx_step(ga, j)).get(sa, sb);
                if (BITS == 4) {
                    if (FOLD) {
                        constexpr uint32_t kMask = 0x000F000Fu, kMagic = 0x43004300u;
                        A[0] = (wv[j] & kMask) | kMagic;
                        A[1] = ((wv[j] >> 4) & kMask) | kMagic;
                        A[2] = ((wv[j] >> 8) & kMask) | kMagic;
                        A[3] = ((wv[j] >> 12) & kMask) | kMagic;
                    } else if (SF32) {
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const float s = (q & 1) ? sb : sa;
                            A[q] = pack_bf2(nibble_centered(wv[j], q) * s,
                                            nibble_centered(wv[j], q + 4) * s);
                        }
                    } else {
                        if (a.fp4)
                            decode_fp4x8(wv[j], A);  // MXFP4: e2m1 values, no zero point
                        else
                            decode_int4(wv[j], A);
                        const __nv_bfloat162 pa = __float2bfloat162_rn(sa);
                        const __nv_bfloat162 pb = __float2bfloat162_rn(sb);
                        const uint32_t ua = *reinterpret_cast<const uint32_t*>(&pa);
                        const uint32_t ub = *reinterpret_cast<const uint32_t*>(&pb);
                        A[0] = bf2_mul(A[0], ua);
                        A[1] = bf2_mul(A[1], ub);
                        A[2] = bf2_mul(A[2], ua);
                        A[3] = bf2_mul(A[3], ub);
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
#pragma unroll
                        for (int m = 0; m < 8; ++m) f[m] *= ((m >> 1) & 1) ? sb : sa;
                    }
#pragma unroll
                    for (int q = 0; q < 4; ++q) A[q] = pack_bf2(f[2 * q], f[2 * q + 1]);
                }
#pragma unroll
                for (int n = 0; n < NT; ++n) {
                    if (SMODE == 1) {
                        if (first && j == 0)
                            mma_bf16_zero(blk[n], A, xa[n][j].x, xa[n][j].y);
                        else
                            mma_bf16(blk[n], A, xa[n][j].x, xa[n][j].y);
                    } else {
                        mma_bf16(acc[n], A, xa[n][j].x, xa[n][j].y);
                    }
                }
            }
        };
        // end of a scale chunk (SMODE 1): undo the fold, scale, accumulate
        auto apply = [&](const ScaleRaw<SF32> sc, const float* csc) {
            float sa, sb;
            sc.get(sa, sb);
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                if (FOLD) {
                    const float2 t = *reinterpret_cast<const float2*>(csc + 8 * n);
                    blk[n][0] = fmaf(-kFoldOffset, t.x, blk[n][0]);
                    blk[n][1] = fmaf(-kFoldOffset, t.y, blk[n][1]);
                    blk[n][2] = fmaf(-kFoldOffset, t.x, blk[n][2]);
                    blk[n][3] = fmaf(-kFoldOffset, t.y, blk[n][3]);
                }
                acc[n][0] = fmaf(sa, blk[n][0], acc[n][0]);
                acc[n][1] = fmaf(sa, blk[n][1], acc[n][1]);
                acc[n][2] = fmaf(sb, blk[n][2], acc[n][2]);
                acc[n][3] = fmaf(sb, blk[n][3], acc[n][3]);
            }
        };

        if (active) {
            const uint8_t* wn = wp + D * GS;                      // loads run D groups ahead
            const uint8_t* xp = xs + r0 * rs + 8 * c;  // this lane's first pair, group 0
            const float* csp = cs + 2 * c;                        // chunk 0, tokens 2c, 2c+1
            int g = 0;  // group relative to g_lo
            // steady rounds: every prefetch is in range
            for (; g + 2 * D <= ng; g += D) {
#pragma unroll
                for (int i = 0; i < D; ++i) {
                    // use slot i, then refill it (no register copy of the old value)
                    group(wr[i], xp + i * KG * 2, sr[0], int(g_lo) + g + i, i % P == 0);
                    wr[i] = ld_stream(wn + i * GS);
                    if (SMODE == 1 && i % P == P - 1) {
                        apply(sr[i / P], csp + (i / P) * ROWS);
                        sr[i / P] = ScaleRaw<SF32>::load(sbase, sidx(int(g_lo) + g + i + 1 - P + D));
                    }
                }
                wn += D * GS;
                xp += D * KG * 2;
                csp += (D / P) * ROWS;
            }
            // drain round: prefetch only what remains
            if (g + D <= ng) {
#pragma unroll
                for (int i = 0; i < D; ++i) {
                    group(wr[i], xp + i * KG * 2, sr[0], int(g_lo) + g + i, i % P == 0);
                    if (g + i + D < ng) wr[i] = ld_stream(wn + i * GS);
                    if (SMODE == 1 && i % P == P - 1) {
                        apply(sr[i / P], csp + (i / P) * ROWS);
                        if (g + i + 1 - P + D < ng)
                            sr[i / P] = ScaleRaw<SF32>::load(sbase, sidx(int(g_lo) + g + i + 1 - P + D));
                    }
                }
                g += D;
                xp += D * KG * 2;
                csp += (D / P) * ROWS;
            }
            // tail: fewer than D groups left, all loaded
#pragma unroll
            for (int i = 0; i < D; ++i) {
                if (g + i < ng) {
                    group(wr[i], xp + i * KG * 2, sr[0], int(g_lo) + g + i, i % P == 0);
                    if (SMODE == 1 && i % P == P - 1) apply(sr[i / P], csp + (i / P) * ROWS);
                }
            }

#pragma unroll
            for (int n = 0; n < NT; ++n) {
                float v[4] = {acc[n][0], acc[n][1], acc[n][2], acc[n][3]};
                if (SMODE == 0) {
                    if (FOLD) {
                        const float2 t = *reinterpret_cast<const float2*>(cs + 8 * n + 2 * c);
                        v[0] = fmaf(-kFoldOffset, t.x, v[0]);
                        v[1] = fmaf(-kFoldOffset, t.y, v[1]);
                        v[2] = fmaf(-kFoldOffset, t.x, v[2]);
                        v[3] = fmaf(-kFoldOffset, t.y, v[3]);
                    }
                    v[0] *= s0;
                    v[1] *= s0;
                    v[2] *= s1;
                    v[3] *= s1;
                }
                epilogue(a, e, rt, r0, c, seg0, M, p0 + 8 * n, v, split, true);
            }
        }
        __syncthreads();  // the next pass restages xs
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
    const int64_t nrb = padded_rows(a.N) / kBlockRows;
    const int64_t rb = blockIdx.x;
    const int64_t rt = rb * kTilesPerBlock + warp;
    if (rt >= nrt) return;
    const int64_t seg0 = a.offsets[e];
    const int M = a.offsets[e + 1] - int(seg0);
    if (M <= 0) return;
    const int64_t ngr = a.K / KG;
    const int64_t nsb = a.block_size > 0 ? a.K / a.block_size : 1;
    int64_t g_lo, g_hi;
    split_range(ngr, a.splits, split, 1, g_lo, g_hi);
    const uint8_t* wtile =
        a.W + (((int64_t)e * nrb + rb) * ngr * kTilesPerBlock + warp) * kUnitBytes + lane * 16;
    constexpr int64_t kGroupStride = (int64_t)kTilesPerBlock * kUnitBytes;
    const int64_t sbase = (((int64_t)e * nrb + rb) * nsb * kTilesPerBlock + warp) * 16 + 2 * r0;
    const float* act = (const float*)a.act;
    const bool sf32 = !a.scale_bf16;

    for (int p0 = 0; p0 < M; p0 += 8) {
        // this lane reduces all 8 tokens of the tile over its k sub-range
        const float* xrow[8];
#pragma unroll
        for (int n = 0; n < 8; ++n) {
            const int tok = min(p0 + n, M - 1);
            const int64_t row = a.rowmap ? a.rowmap[seg0 + tok] : seg0 + tok;
            xrow[n] = act + row * a.K;
        }
        float acc[8][2];
#pragma unroll
        for (int n = 0; n < 8; ++n) acc[n][0] = acc[n][1] = 0.0f;
        for (int64_t g = g_lo; g < g_hi; ++g) {
            const uint4 w = *reinterpret_cast<const uint4*>(wtile + g * kGroupStride);
            const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
            // decode the lane's 2 x KL codes into (row, actual k) order
            float q[2][KL];
            // q[row][4j + t] is the code at k = 16j + 4c + t of row r0 (+8)
            if (BITS == 4) {
#pragma unroll
                for (int j = 0; j < 4; ++j)
#pragma unroll
                    for (int p = 0; p < 8; ++p)
                        q[p & 1][4 * j + 2 * ((p >> 1) & 1) + (p >> 2)] =
                            a.fp4 ? fp4_to_float(wv[j] >> (4 * p)) : nibble_centered(wv[j], p);
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
            // the lane's k values span several blocks when block_size < KG: one
            // scale per 4-wide run (block_size >= 16 keeps each run in one block)
#pragma unroll
            for (int j = 0; j < KL / 4; ++j) {
                const int64_t kk = g * KG + 16 * j + 4 * c;
                const int64_t b = a.block_size > 0 ? kk / a.block_size : 0;
                const float sa = load_scale(a.S, sbase + b * 128, sf32);
                const float sb = load_scale(a.S, sbase + b * 128 + 1, sf32);
#pragma unroll
                for (int n = 0; n < 8; ++n) {
                    const float4 xv = *reinterpret_cast<const float4*>(xrow[n] + kk);
                    const float xs[4] = {xv.x, xv.y, xv.z, xv.w};
                    float pa = 0.0f, pb = 0.0f;
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        pa = fmaf(q[0][4 * j + u], xs[u], pa);
                        pb = fmaf(q[1][4 * j + u], xs[u], pb);
                    }
                    acc[n][0] = fmaf(sa, pa, acc[n][0]);
                    acc[n][1] = fmaf(sb, pb, acc[n][1]);
                }
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
        epilogue(a, e, rt, r0, c, seg0, M, p0, v, split, false);
    }
}

template <int BITS, int SMODE, bool SF32, int NT, int P>
cudaError_t launch_one(const FfnArgs& a, dim3 grid, size_t smem, cudaStream_t st) {
    return launch_kernel(ffn_decode_kernel<BITS, SMODE, SF32, NT, P>, grid, dim3(kWarps * 32), smem, st, a.pdl != 0,
                         a);
}

template <int BITS, int SMODE, bool SF32, int P>
cudaError_t launch_nt(const FfnArgs& a, dim3 grid, size_t smem, cudaStream_t st) {
    switch (a.nt) {
        case 1: return launch_one<BITS, SMODE, SF32, 1, P>(a, grid, smem, st);
        case 2: return launch_one<BITS, SMODE, SF32, 2, P>(a, grid, smem, st);
        default: return launch_one<BITS, SMODE, SF32, 4, P>(a, grid, smem, st);
    }
}

template <int BITS, int SMODE, int P>
cudaError_t launch_sf(const FfnArgs& a, dim3 grid, size_t smem, cudaStream_t st) {
    return a.scale_bf16 ? launch_nt<BITS, SMODE, false, P>(a, grid, smem, st)
                        : launch_nt<BITS, SMODE, true, P>(a, grid, smem, st);
}

template <int BITS, int SMODE, bool SF32, int P>
cudaError_t raise_smem_nt() {
    const int lim = int(kDecodeSmemLimit);
    cudaError_t e = cudaFuncSetAttribute(ffn_decode_kernel<BITS, SMODE, SF32, 1, P>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(ffn_decode_kernel<BITS, SMODE, SF32, 2, P>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(ffn_decode_kernel<BITS, SMODE, SF32, 4, P>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
    return e;
}

template <int BITS, int SMODE, int P>
cudaError_t raise_smem_sf() {
    cudaError_t e = raise_smem_nt<BITS, SMODE, false, P>();
    return e == cudaSuccess ? raise_smem_nt<BITS, SMODE, true, P>() : e;
}

// groups per scale application for SMODE 1
int chunk_groups(int bits, int block_size) {
    const int gpb = block_size / kgroup_of(bits);
    return gpb >= kRing ? kRing : gpb;
}

}  // namespace

int64_t decode_smem_bytes(int64_t K, int bits, int block_size, int splits, int nt) {
    const int kg = kgroup_of(bits);
    const int64_t ngr = K / kg;
    const int64_t gpb = (block_size >= kg) ? block_size / kg : 1;
    const int64_t nblk = (ngr + gpb - 1) / gpb;
    const int64_t per = (nblk + splits - 1) / splits;
    const int64_t groups = std::min<int64_t>(ngr, per * gpb);
    const int64_t sums = (block_size >= kg) ? groups / chunk_groups(bits, block_size) : 1;
    return int64_t(8) * nt * (staged_row_bytes(groups * kg) + 4 * sums);
}

cudaError_t prepare_ffn_decode() {
    cudaError_t e = cudaSuccess;
    if (e == cudaSuccess) e = raise_smem_sf<4, 0, 1>();
    if (e == cudaSuccess) e = raise_smem_sf<4, 1, 1>();
    if (e == cudaSuccess) e = raise_smem_sf<4, 1, 2>();
    if (e == cudaSuccess) e = raise_smem_sf<4, 1, 4>();
    if (e == cudaSuccess) e = raise_smem_sf<4, 1, 8>();
    if (e == cudaSuccess) e = raise_smem_sf<4, 2, 1>();
    if (e == cudaSuccess) e = raise_smem_sf<8, 0, 1>();
    if (e == cudaSuccess) e = raise_smem_sf<8, 1, 1>();
    if (e == cudaSuccess) e = raise_smem_sf<8, 1, 2>();
    if (e == cudaSuccess) e = raise_smem_sf<8, 1, 4>();
    if (e == cudaSuccess) e = raise_smem_sf<8, 1, 8>();
    if (e == cudaSuccess) e = raise_smem_sf<8, 2, 1>();
    return e;
}

int scale_mode(int bits, int block_size) {
    if (block_size == 0) return 0;
    return block_size >= kgroup_of(bits) ? 1 : 2;
}

cudaError_t launch_ffn_decode(const FfnArgs& a, cudaStream_t st) {
    dim3 grid(unsigned(padded_rows(a.N) / kBlockRows), unsigned(a.E), unsigned(a.splits));
    const size_t smem = size_t(decode_smem_bytes(a.K, a.bits, a.block_size, a.splits, a.nt));
    if (smem > kDecodeSmemLimit) return cudaErrorInvalidConfiguration;
    const int sm = scale_mode(a.bits, a.block_size);
    const int P = sm == 1 ? chunk_groups(a.bits, a.block_size) : 1;
    if (a.bits == 4) {
        if (sm == 0) return launch_sf<4, 0, 1>(a, grid, smem, st);
        if (sm == 2) return launch_sf<4, 2, 1>(a, grid, smem, st);
        if (P == 1) return launch_sf<4, 1, 1>(a, grid, smem, st);
        if (P == 2) return launch_sf<4, 1, 2>(a, grid, smem, st);
        if (P == 4) return launch_sf<4, 1, 4>(a, grid, smem, st);
        return launch_sf<4, 1, 8>(a, grid, smem, st);
    }
    if (sm == 0) return launch_sf<8, 0, 1>(a, grid, smem, st);
    if (sm == 2) return launch_sf<8, 2, 1>(a, grid, smem, st);
    if (P == 1) return launch_sf<8, 1, 1>(a, grid, smem, st);
    if (P == 2) return launch_sf<8, 1, 2>(a, grid, smem, st);
    if (P == 4) return launch_sf<8, 1, 4>(a, grid, smem, st);
    return launch_sf<8, 1, 8>(a, grid, smem, st);
}

cudaError_t launch_ffn_simt(const FfnArgs& a, cudaStream_t st) {
    dim3 grid(unsigned(padded_rows(a.N) / kBlockRows), unsigned(a.E), unsigned(a.splits));
    if (a.bits == 4)
        ffn_simt_kernel<4><<<grid, kWarps * 32, 0, st>>>(a);
    else
        ffn_simt_kernel<8><<<grid, kWarps * 32, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace qmoe
