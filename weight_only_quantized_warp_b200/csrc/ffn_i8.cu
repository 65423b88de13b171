// ffn_i8.cu -- the int8 block compute tier of the expert FFN layers.
//
// "ClikaRT::nn::QMoEWoQ" (class description): a packed block weight on the
// int8 block tier takes its activation rounded to per-block int8 before the
// dot. The pages give no rounding rule; it is read as symmetric absmax
// rounding over the weight's own K blocks, decided in fp32:
//   s = absmax(block) / 127, q = clamp(rint(v / s), -127, 127), ties to even
//   (s = 0, q = 0 for an all-zero block),
// and the dot of one weight row as the sum over blocks of
//   s_w * s * sum_k (c_k - z) q_k
// with the stored unsigned weight code c and its zero point z = 2^(bits-1).
//
// quantize_rows_i8_kernel rounds activation rows (x, the router-weighted
// rows, or h) into codes and per-block scales. ffn_i8_kernel streams the
// packed weights exactly like the bf16 decode kernels (same fragment-order
// layout, CTA per 128-row block, warp per 16-row tile, ring of 16-byte loads,
// staged activation rows) but feeds the codes to the integer MMA m16n8k32 with
// u8 weights -- the codes as stored, no decode to floating point -- and s8
// activations, accumulating exact int32 per scale chunk. The zero point comes
// off after the MMA: sum_k (c_k - z) q_k = sum_k c_k q_k - z * sum_k q_k, with
// the activation code sums per chunk computed once per CTA pass from the
// staged codes (dp4a).
//
// Fragments of m16n8k32 (8-bit operands): lane L holds A registers (row r0,
// k 4c..4c+3), (row r0+8, same), (row r0, k 16+4c..16+4c+3), (row r0+8, same)
// with r0 = L/4, c = L%4, four codes per register in increasing k; B
// registers (k 4c..4c+3, column r0) and (k 16+4c.., column r0); C rows r0 and
// r0 + 8 at columns 2c, 2c+1. The packed weight words already hold, per lane,
// the codes of rows r0 and r0 + 8 at k = 16j + 4c + {0..3} (word j for 4-bit
// codes, word pair 2j, 2j+1 for 8-bit codes):
//   4-bit: the low nibbles of word j (w & 0x0F0F0F0F) are row r0's codes at
//     k + {0, 2, 1, 3} in byte order and the high nibbles (w >> 4, same mask)
//     row r0 + 8's, so one MMA takes words 2m and 2m + 1 of the group with
//     two bit operations and one shift per word; the activation codes are
//     stored with the same swap of the middle two bytes of every 4-code run,
//     so that both operands pair the same k;
//   8-bit: bytes 0, 1 of word 2j and bytes 0, 1 of word 2j + 1 are row r0's
//     codes at k + 0..3 and bytes 2, 3 of each row r0 + 8's, so one byte
//     permute per register gives them in natural order.
#include <algorithm>

#include "qmoe_internal.cuh"
#include "stream_common.cuh"

namespace qmoe {
namespace {

constexpr int kWarps = 8;
constexpr int kRing = 8;       // weight loads in flight per lane
constexpr int kMaxChunk = 8;   // k-groups per scale chunk at most (the kernels built)

// D (int32) = A (u8) x B (s8) [+ D]
__device__ __forceinline__ void mma_u8s8(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_u8s8_zero(int (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                              uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%10,%10,%10,%10};"
        : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "r"(0));
}

// ------------------------------------------------------------ quantisation

// One warp per (row, span of max(bs, 128) codes): lane l covers codes
// 4l .. 4l + 3 of every 128-code step of the span; a block of bs < 128 codes
// is bs / 4 consecutive lanes. Pass 1 finds the block's absmax, pass 2
// writes the codes (one 32-bit word per lane and step) and lane 0 of the
// block its scale.
// LAYOUT: 0 natural order; 1 the middle two codes of every run of 4 swapped
// (k + {0, 2, 1, 3}: the nibble order of 4-bit weight words, for
// ffn_i8_kernel); 2 and 3 the tensor-core order of ffn_tc_i8_kernel: within
// every 32-code chunk, the run of codes k = 4 r .. 4 r + 3 goes to run
// 2 (r % 4) + r / 4, with the middle two codes swapped (2, 4-bit weights) or
// not (3, 8-bit weights).
template <bool IN_BF16, int LAYOUT>
__global__ void __launch_bounds__(256) quantize_rows_i8_kernel(const void* x, int64_t rows, int64_t K, int bs,
                                                               int8_t* q, float* s) {
    const int lane = threadIdx.x & 31;
    const int64_t unit = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t span = bs > 128 ? bs : 128;
    const int64_t per_row = (K + span - 1) / span;
    if (unit >= rows * per_row) return;  // uniform over the warp
    const int64_t row = unit / per_row;
    const int64_t k0 = (unit - row * per_row) * span;
    const int steps = int(span / 128);
    const int G = (bs < 128 ? bs : 128) / 4;  // lanes of one block in a step

    auto load4 = [&](int64_t k, float (&v)[4]) {
        if (k >= K) {
            v[0] = v[1] = v[2] = v[3] = 0.0f;
        } else if (IN_BF16) {
            const uint2 u = *reinterpret_cast<const uint2*>((const __nv_bfloat16*)x + row * K + k);
            v[0] = __uint_as_float(u.x << 16);
            v[1] = __uint_as_float(u.x & 0xFFFF0000u);
            v[2] = __uint_as_float(u.y << 16);
            v[3] = __uint_as_float(u.y & 0xFFFF0000u);
        } else {
            const float4 f = *reinterpret_cast<const float4*>((const float*)x + row * K + k);
            v[0] = f.x;
            v[1] = f.y;
            v[2] = f.z;
            v[3] = f.w;
        }
    };

    float amax = 0.0f;
    for (int st = 0; st < steps; ++st) {
        float v[4];
        load4(k0 + st * 128 + lane * 4, v);
#pragma unroll
        for (int i = 0; i < 4; ++i) amax = fmaxf(amax, fabsf(v[i]));
    }
    for (int o = G / 2; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float sc = __fdiv_rn(amax, 127.0f);

    for (int st = 0; st < steps; ++st) {
        const int64_t k = k0 + st * 128 + lane * 4;
        if (k >= K) break;
        float v[4];
        load4(k, v);
        uint32_t b[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            int c = sc > 0.0f ? __float2int_rn(__fdiv_rn(v[i], sc)) : 0;
            c = max(-127, min(127, c));
            b[i] = uint32_t(c) & 0xFFu;
        }
        constexpr bool SWAP = LAYOUT == 1 || LAYOUT == 2;
        const uint32_t word = SWAP ? (b[0] | (b[2] << 8) | (b[1] << 16) | (b[3] << 24))
                                   : (b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24));
        int64_t kout = k;
        if (LAYOUT >= 2) {
            const int rq = lane & 7;  // run of 4 inside the lane's 32-code chunk
            kout = k - 4 * rq + 4 * (2 * (rq & 3) + (rq >> 2));
        }
        *reinterpret_cast<uint32_t*>(q + row * K + kout) = word;
    }
    const int64_t kl = k0 + lane * 4;
    if ((lane & (G - 1)) == 0 && kl < K) s[row * (K / bs) + kl / bs] = sc;
}

// ------------------------------------------------------------- expert FFN

// Bytes of one staged row of kr activation codes: 16 bytes of padding make
// the row stride an odd multiple of 16 bytes (kr is a multiple of 32), so the
// 32-bit reads of rows r0 = 0..7 at offsets 4c land in 32 distinct banks.
__host__ __device__ constexpr int64_t staged_row_bytes_i8(int64_t kr) { return kr + 16; }

// P: k-groups per scale chunk (min(groups per block, kMaxChunk)); the chunk's
// int32 partial is scaled and added to the fp32 accumulator at its end.
//
// One CTA = 8 warps = the 8 row tiles of one 128-row block of one expert, for
// one K-split; passes of 8*NT rows of the expert's segment. The k-group loop
// has a steady part (loads always in range), one guarded drain round and a
// tail, as in the bf16 decode kernels.
template <int BITS, bool SF32, int NT, int P>
__global__ void __launch_bounds__(kWarps * 32, NT == 1 ? 3 : 2) ffn_i8_kernel(const FfnArgs a) {
    constexpr int KG = kgroup_of(BITS);
    constexpr int D = kRing;
    static_assert(D % P == 0, "scale chunk must divide the ring");
    constexpr int GS = kTilesPerBlock * kUnitBytes;  // group stride, 4 KB
    constexpr int ROWS = 8 * NT;
    constexpr int LG_KG = BITS == 4 ? 6 : 5;
    constexpr int CK = P * KG;  // codes per chunk
    extern __shared__ __align__(16) uint8_t xs[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int r0 = lane >> 2, c = lane & 3;
    const int e = blockIdx.y, split = blockIdx.z;
    const int64_t rb = blockIdx.x;
    const int64_t nrt = a.N / kTileRows;
    const int64_t nrb = padded_rows(a.N) / kBlockRows;
    const int64_t rt = rb * kTilesPerBlock + warp;
    const bool active = rt < nrt;
    const int64_t seg0 = a.offsets[e];
    const int M = a.offsets[e + 1] - int(seg0);
    if (M <= 0) return;  // uniform over the CTA
    const int64_t ngr = a.K / KG;
    const int64_t nsb = a.K / a.block_size;
    const int lg_gpb = (__ffs(a.block_size) - 1) - LG_KG;
    int64_t g_lo, g_hi;
    split_range(ngr, a.splits, split, int64_t(1) << lg_gpb, g_lo, g_hi);
    const int ng = int(g_hi - g_lo);
    const int kr = ng * KG;
    const int rs = int(staged_row_bytes_i8(kr));
    const int chunks16 = kr / 16;
    const int nch = ng / P;
    // per (chunk, row): {activation scale of the chunk's block, z * code sum}
    float2* ct = reinterpret_cast<float2*>(xs + ROWS * rs);

    const uint8_t* wp =
        a.W + (((int64_t)e * nrb + rb) * ngr * kTilesPerBlock + warp) * kUnitBytes + lane * 16 +
        g_lo * GS;
    const int64_t sb0 = (((int64_t)e * nrb + rb) * nsb * kTilesPerBlock + warp) * 16 + 2 * r0;
    const void* sbase = SF32 ? (const void*)((const float*)a.S + sb0)
                             : (const void*)((const __nv_bfloat16*)a.S + sb0);
    auto sidx = [&](int ga) -> int { return (ga >> lg_gpb) * 128; };

    for (int p0 = 0; p0 < M; p0 += ROWS) {
        uint4 wr[D];
        ScaleRaw<SF32> sr[D / P];
        if (active) {
#pragma unroll
            for (int i = 0; i < D; ++i) {
                if (i < ng) {
                    wr[i] = ld_stream(wp + i * GS);
                    if (i % P == 0) sr[i / P] = ScaleRaw<SF32>::load(sbase, sidx(int(g_lo) + i));
                }
            }
        }
        // stage the code rows of tokens p0 .. p0 + ROWS - 1 (clamped)
        for (int row = warp; row < ROWS; row += kWarps) {
            const int tok = min(p0 + row, M - 1);
            const int64_t srow = a.rowmap ? a.rowmap[seg0 + tok] : seg0 + tok;
            const int8_t* src = a.aq + srow * a.K + g_lo * KG;
            uint8_t* dst = xs + row * rs;
            for (int ch = lane; ch < chunks16; ch += 32) cp_async16(dst + ch * 16, src + ch * 16);
        }
        cp_async_wait_all();
        __syncthreads();
        // chunk table: one thread per (chunk, row)
        for (int i = tid; i < nch * ROWS; i += blockDim.x) {
            const int b = i / ROWS, row = i - b * ROWS;
            const uint4* src = reinterpret_cast<const uint4*>(xs + row * rs + b * CK);
            int sum = 0;
#pragma unroll 4
            for (int u = 0; u < CK / 16; ++u) {
                const uint4 v = src[u];
                sum = __dp4a(int(v.x), 0x01010101, sum);
                sum = __dp4a(int(v.y), 0x01010101, sum);
                sum = __dp4a(int(v.z), 0x01010101, sum);
                sum = __dp4a(int(v.w), 0x01010101, sum);
            }
            const int tok = min(p0 + row, M - 1);
            const int64_t srow = a.rowmap ? a.rowmap[seg0 + tok] : seg0 + tok;
            const float sx = a.as[srow * nsb + ((g_lo + int64_t(b) * P) >> lg_gpb)];
            ct[i] = make_float2(sx, __int_as_float(sum << (BITS - 1)));
        }
        __syncthreads();

        float acc[NT][4];
        int blk[NT][4];
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                acc[n][q] = 0.0f;
                blk[n][q] = 0;
            }

        // one k-group: xg is this lane's first activation word of the group
        // (row r0, byte 4c); first: the group opens a scale chunk
        auto group = [&](const uint4 w, const uint8_t* xg, bool first) {
            const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
            if (BITS == 4) {
                uint32_t xb[NT][4];
#pragma unroll
                for (int n = 0; n < NT; ++n)
#pragma unroll
                    for (int j = 0; j < 4; ++j) xb[n][j] = *reinterpret_cast<const uint32_t*>(xg + n * 8 * rs + 16 * j);
                constexpr uint32_t kLo = 0x0F0F0F0Fu;
#pragma unroll
                for (int m = 0; m < 2; ++m) {
                    const uint32_t A[4] = {wv[2 * m] & kLo, (wv[2 * m] >> 4) & kLo, wv[2 * m + 1] & kLo,
                                           (wv[2 * m + 1] >> 4) & kLo};
#pragma unroll
                    for (int n = 0; n < NT; ++n) {
                        if (first && m == 0)
                            mma_u8s8_zero(blk[n], A, xb[n][2 * m], xb[n][2 * m + 1]);
                        else
                            mma_u8s8(blk[n], A, xb[n][2 * m], xb[n][2 * m + 1]);
                    }
                }
            } else {
                uint32_t xb[NT][2];
#pragma unroll
                for (int n = 0; n < NT; ++n)
#pragma unroll
                    for (int j = 0; j < 2; ++j) xb[n][j] = *reinterpret_cast<const uint32_t*>(xg + n * 8 * rs + 16 * j);
                const uint32_t A[4] = {__byte_perm(wv[0], wv[1], 0x5410), __byte_perm(wv[0], wv[1], 0x7632),
                                       __byte_perm(wv[2], wv[3], 0x5410), __byte_perm(wv[2], wv[3], 0x7632)};
#pragma unroll
                for (int n = 0; n < NT; ++n) {
                    if (first)
                        mma_u8s8_zero(blk[n], A, xb[n][0], xb[n][1]);
                    else
                        mma_u8s8(blk[n], A, xb[n][0], xb[n][1]);
                }
            }
        };
        // end of a scale chunk: remove the zero point, scale, accumulate
        auto apply = [&](const ScaleRaw<SF32> sc, const float2* cst) {
            float sa, sb;
            sc.get(sa, sb);
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                const float4 t = *reinterpret_cast<const float4*>(cst + 8 * n + 2 * c);
                const float d0 = float(blk[n][0] - __float_as_int(t.y));
                const float d1 = float(blk[n][1] - __float_as_int(t.w));
                const float d2 = float(blk[n][2] - __float_as_int(t.y));
                const float d3 = float(blk[n][3] - __float_as_int(t.w));
                acc[n][0] = fmaf(sa * t.x, d0, acc[n][0]);
                acc[n][1] = fmaf(sa * t.z, d1, acc[n][1]);
                acc[n][2] = fmaf(sb * t.x, d2, acc[n][2]);
                acc[n][3] = fmaf(sb * t.z, d3, acc[n][3]);
            }
        };

        if (active) {
            const uint8_t* wn = wp + D * GS;          // loads run D groups ahead
            const uint8_t* xp = xs + r0 * rs + 4 * c;  // this lane's first word, group 0
            const float2* csp = ct;                    // chunk 0
            int g = 0;                                 // group relative to g_lo
            for (; g + 2 * D <= ng; g += D) {
#pragma unroll
                for (int i = 0; i < D; ++i) {
                    group(wr[i], xp + i * KG, i % P == 0);
                    wr[i] = ld_stream(wn + i * GS);
                    if (i % P == P - 1) {
                        apply(sr[i / P], csp + (i / P) * ROWS);
                        sr[i / P] = ScaleRaw<SF32>::load(sbase, sidx(int(g_lo) + g + i + 1 - P + D));
                    }
                }
                wn += D * GS;
                xp += D * KG;
                csp += (D / P) * ROWS;
            }
            if (g + D <= ng) {
#pragma unroll
                for (int i = 0; i < D; ++i) {
                    group(wr[i], xp + i * KG, i % P == 0);
                    if (g + i + D < ng) wr[i] = ld_stream(wn + i * GS);
                    if (i % P == P - 1) {
                        apply(sr[i / P], csp + (i / P) * ROWS);
                        if (g + i + 1 - P + D < ng)
                            sr[i / P] = ScaleRaw<SF32>::load(sbase, sidx(int(g_lo) + g + i + 1 - P + D));
                    }
                }
                g += D;
                xp += D * KG;
                csp += (D / P) * ROWS;
            }
#pragma unroll
            for (int i = 0; i < D; ++i) {
                if (g + i < ng) {
                    group(wr[i], xp + i * KG, i % P == 0);
                    if (i % P == P - 1) apply(sr[i / P], csp + (i / P) * ROWS);
                }
            }
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                const float v[4] = {acc[n][0], acc[n][1], acc[n][2], acc[n][3]};
                epilogue(a, e, rt, r0, c, seg0, M, p0 + 8 * n, v, split, a.act_bf16 != 0);
            }
        }
        __syncthreads();  // the next pass restages xs
    }
}

template <int BITS, bool SF32, int NT, int P>
cudaError_t launch_one(const FfnArgs& a, dim3 grid, size_t smem, cudaStream_t st) {
    ffn_i8_kernel<BITS, SF32, NT, P><<<grid, kWarps * 32, smem, st>>>(a);
    return cudaGetLastError();
}

template <int BITS, bool SF32, int P>
cudaError_t launch_nt(const FfnArgs& a, dim3 grid, size_t smem, cudaStream_t st) {
    switch (a.nt) {
        case 1: return launch_one<BITS, SF32, 1, P>(a, grid, smem, st);
        case 2: return launch_one<BITS, SF32, 2, P>(a, grid, smem, st);
        default: return launch_one<BITS, SF32, 4, P>(a, grid, smem, st);
    }
}

template <int BITS, int P>
cudaError_t launch_sf(const FfnArgs& a, dim3 grid, size_t smem, cudaStream_t st) {
    return a.scale_bf16 ? launch_nt<BITS, false, P>(a, grid, smem, st) : launch_nt<BITS, true, P>(a, grid, smem, st);
}

template <int BITS, bool SF32, int P>
cudaError_t raise_nt() {
    const int lim = int(kDecodeSmemLimit);
    cudaError_t e = cudaFuncSetAttribute(ffn_i8_kernel<BITS, SF32, 1, P>, cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(ffn_i8_kernel<BITS, SF32, 2, P>, cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(ffn_i8_kernel<BITS, SF32, 4, P>, cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
    return e;
}

template <int BITS, int P>
cudaError_t raise_sf() {
    cudaError_t e = raise_nt<BITS, false, P>();
    return e == cudaSuccess ? raise_nt<BITS, true, P>() : e;
}

int chunk_groups(int bits, int block_size) {
    const int gpb = block_size / kgroup_of(bits);
    return gpb >= kMaxChunk ? kMaxChunk : gpb;
}

}  // namespace

int64_t i8_smem_bytes(int64_t K, int bits, int block_size, int splits, int nt) {
    const int kg = kgroup_of(bits);
    const int64_t ngr = K / kg;
    const int64_t gpb = block_size / kg;
    const int64_t nblk = (ngr + gpb - 1) / gpb;
    const int64_t per = (nblk + splits - 1) / splits;
    const int64_t groups = std::min<int64_t>(ngr, per * gpb);
    const int64_t chunks = groups / chunk_groups(bits, block_size);
    return int64_t(8) * nt * (staged_row_bytes_i8(groups * kg) + 8 * chunks);
}

cudaError_t prepare_ffn_i8() {
    cudaError_t e = cudaSuccess;
    if (e == cudaSuccess) e = raise_sf<4, 1>();
    if (e == cudaSuccess) e = raise_sf<4, 2>();
    if (e == cudaSuccess) e = raise_sf<4, 4>();
    if (e == cudaSuccess) e = raise_sf<4, 8>();
    if (e == cudaSuccess) e = raise_sf<8, 1>();
    if (e == cudaSuccess) e = raise_sf<8, 2>();
    if (e == cudaSuccess) e = raise_sf<8, 4>();
    if (e == cudaSuccess) e = raise_sf<8, 8>();
    return e;
}

cudaError_t launch_ffn_i8(const FfnArgs& a, cudaStream_t st) {
    if (a.block_size < kgroup_of(a.bits) || !a.aq || !a.as) return cudaErrorInvalidValue;
    dim3 grid(unsigned(padded_rows(a.N) / kBlockRows), unsigned(a.E), unsigned(a.splits));
    const size_t smem = size_t(i8_smem_bytes(a.K, a.bits, a.block_size, a.splits, a.nt));
    if (smem > kDecodeSmemLimit) return cudaErrorInvalidConfiguration;
    const int P = chunk_groups(a.bits, a.block_size);
    if (a.bits == 4) {
        if (P == 1) return launch_sf<4, 1>(a, grid, smem, st);
        if (P == 2) return launch_sf<4, 2>(a, grid, smem, st);
        if (P == 4) return launch_sf<4, 4>(a, grid, smem, st);
        return launch_sf<4, 8>(a, grid, smem, st);
    }
    if (P == 1) return launch_sf<8, 1>(a, grid, smem, st);
    if (P == 2) return launch_sf<8, 2>(a, grid, smem, st);
    if (P == 4) return launch_sf<8, 4>(a, grid, smem, st);
    return launch_sf<8, 8>(a, grid, smem, st);
}

template <bool IN_BF16>
void launch_quantize_layout(int layout, unsigned grid, const void* x, int64_t rows, int64_t K, int bs, int8_t* q,
                            float* s, cudaStream_t st) {
    switch (layout) {
        case 1: quantize_rows_i8_kernel<IN_BF16, 1><<<grid, 256, 0, st>>>(x, rows, K, bs, q, s); break;
        case 2: quantize_rows_i8_kernel<IN_BF16, 2><<<grid, 256, 0, st>>>(x, rows, K, bs, q, s); break;
        case 3: quantize_rows_i8_kernel<IN_BF16, 3><<<grid, 256, 0, st>>>(x, rows, K, bs, q, s); break;
        default: quantize_rows_i8_kernel<IN_BF16, 0><<<grid, 256, 0, st>>>(x, rows, K, bs, q, s); break;
    }
}

cudaError_t launch_quantize_i8(const void* x, int act_bf16, int64_t rows, int64_t K, int bs, int layout, int8_t* q,
                               float* s, cudaStream_t st) {
    if (rows <= 0) return cudaSuccess;
    const int64_t span = bs > 128 ? bs : 128;
    const int64_t warps = rows * ((K + span - 1) / span);
    const unsigned grid = unsigned((warps + 7) / 8);
    if (act_bf16)
        launch_quantize_layout<true>(layout, grid, x, rows, K, bs, q, s, st);
    else
        launch_quantize_layout<false>(layout, grid, x, rows, K, bs, q, s, st);
    return cudaGetLastError();
}

}  // namespace qmoe
