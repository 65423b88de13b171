// ffn_stream.cu -- expert FFN layers for few routed rows per expert: the
// packed weights stream from HBM through a shared-memory ring.
//
// Each linear is y = x @ dequant(W).T + b ("QLinearWoQ" page, class summary)
// over the rows routed to one expert, the weights decoded block by block
// inside the dot and never written out dense ("ClikaRT::nn::QMoEWoQ", class
// description); FC1 applies the gated activation of the QMoE page in its
// epilogue. With a few rows per expert the layer is bound by reading the
// packed weights once, so this kernel is built around that stream:
//
//   * one persistent CTA per SM takes a contiguous run of work items
//     (touched expert, K split, 128-row block; row block fastest), so its
//     items share their activation rows, which it stages once in shared
//     memory with their per-group sums;
//   * warp 16 streams the item's packed codes, one 4 KB slab per k-group of
//     the 128-row block (the pack keeps a slab contiguous), through a ring of
//     up to 16 slabs with cp.async.bulk and an mbarrier per slab: up to 64 KB
//     per SM in flight, held by shared memory rather than registers;
//   * warps 0-15 consume: warp w decodes row tile w % 8 of the k-groups of
//     parity w / 8 from the ring (one 16-byte read per lane), runs the
//     m16n8k16 MMAs against the staged rows and releases the slab; the two
//     warps of a tile add their halves at the end of the item.
//
// Fragments, the OR-magic int4 decode with the zero point folded out after
// the MMA, the exact int8 decode and the scale handling per k-group are those
// of ffn_decode.cu (which keeps the kernels for blocks smaller than a k-group
// and for MXFP4 codes). Every wait is bounded (about four seconds): a wait
// that runs out raises the CTA's abort flag and QMOE_TIMEOUT in the status
// word, and every role then finishes its loops without work, so the CTA
// always reaches its barriers and exits.
#include <algorithm>

#include "qmoe_internal.cuh"
#include "stream_common.cuh"

namespace qmoe {
namespace {

constexpr int kSCons = 16;                      // consumer warps
constexpr int kSThreads = (kSCons + 1) * 32;    // plus the producer warp
constexpr int kSSlab = kTilesPerBlock * kUnitBytes;  // one k-group of a 128-row block, 4 KB
constexpr int kSStagesMax = 16;
constexpr int kSBarBytes = 1024;

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_bf16_zero(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%10,%10,%10,%10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.0f));
}

__device__ __forceinline__ uint32_t pack_bf2(float lo, float hi) {
    __nv_bfloat162 r = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&r);
}

// byte m of w -> fp32 (q - 128), exactly: 0x4B000000 is 2^23 with unit 1
__device__ __forceinline__ float byte_centered(uint32_t w, int m) {
    return __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7440u | m)) - 8388736.0f;
}

__device__ __forceinline__ uint32_t s_addr(const void* p) { return uint32_t(__cvta_generic_to_shared(p)); }

__device__ __forceinline__ void sbar_init(uint32_t bar, uint32_t n) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(n));
}
__device__ __forceinline__ void sbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void sbar_expect(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
// potentially blocking test: the warp sleeps up to 20 us while the phase is open
__device__ __forceinline__ bool sbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\nselp.b32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(20000u)
        : "memory");
    return ok != 0;
}
// Bounded wait: false after about four seconds (the abort flag and the
// status word are then raised) or once another warp has aborted.
__device__ __forceinline__ bool sbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag, int32_t* status) {
    for (int it = 0; it < 200000; ++it) {
        if (sbar_try(bar, parity)) return true;
        if (*abort_flag) return false;
    }
    *abort_flag = 1;
    atomicExch(status, int32_t(QMOE_TIMEOUT));
    return false;
}
__device__ __forceinline__ void bulk_slab(uint32_t dst, const void* src, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(uint32_t(kSSlab)), "r"(bar)
                 : "memory");
}
// barrier among the 16 consumer warps only (the producer never joins)
__device__ __forceinline__ void consumers_sync() { asm volatile("bar.sync 1, 512;" ::: "memory"); }

// Shared memory of one CTA: the slab ring and its barriers, the two warps'
// partial exchange, the staged rows (8 * NT of them, kr k-values each,
// padded by 32 bytes so 8-byte reads of 4 rows x 4 lanes hit distinct banks)
// and their sums (per k-group and row for block scales, per row otherwise).
__host__ __device__ constexpr int64_t stream_row_bytes(int64_t kr) { return kr * 2 + 32; }

struct StreamLayout {
    int64_t ring, bars, xch, rows, sums, total;
};

__host__ __device__ inline StreamLayout stream_layout(int64_t kr_max, int ng_max, int nt, int stages) {
    StreamLayout L{};
    L.ring = 0;
    L.bars = L.ring + int64_t(stages) * kSSlab;
    L.xch = L.bars + kSBarBytes;
    L.rows = L.xch + int64_t(kTilesPerBlock) * 32 * 4 * nt * 4;
    L.sums = L.rows + int64_t(8) * nt * stream_row_bytes(kr_max);
    L.total = L.sums + int64_t(8) * nt * ng_max * 4;
    return L;
}

constexpr float kFold = 136.0f;  // 128 (the bf16 magic) + 8 (the int4 zero point)

// Work item i of the CTA's run: touched expert (in id order), K split, row block.
struct SItem {
    int e, split, rb;
};

__device__ __forceinline__ SItem stream_item(int i, int nrb, int splits, const int* touched_ids) {
    SItem it;
    const int per_e = nrb * splits;
    const int te = i / per_e;
    const int rem = i - te * per_e;
    it.e = touched_ids[te];
    it.split = rem / nrb;
    it.rb = rem - it.split * nrb;
    return it;
}

// SMODE 0: one scale per row (applied after the K range); 1: block scales of
// one k-group or more (applied per k-group). NT: 8-token MMA tiles per pass.
template <int BITS, int SMODE, bool SF32, int NT>
__global__ void __launch_bounds__(kSThreads, 1) ffn_stream_kernel(const FfnArgs a, int32_t* status, int stages) {
    constexpr int KG = kgroup_of(BITS);
    constexpr int KSTEPS = BITS == 4 ? 4 : 2;
    constexpr int LG_KG = BITS == 4 ? 6 : 5;
    constexpr bool FOLD = BITS == 4;
    constexpr int ROWS = 8 * NT;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    const int nrb = int(padded_rows(a.N) / kBlockRows);
    const int64_t nrt = a.N / kTileRows;
    const int64_t ngr = a.K / KG;
    const int64_t nsb = a.block_size > 0 ? a.K / a.block_size : 1;
    const int lg_gpb = SMODE == 1 ? (__ffs(a.block_size) - 1) - LG_KG : 0;
    const int gpb = 1 << lg_gpb;
    // the largest k range of a split
    int64_t g0, g1;
    split_range(ngr, a.splits, 0, gpb, g0, g1);
    const int ng_max = int(g1 - g0);
    const StreamLayout L = stream_layout(ng_max * KG, ng_max, NT, stages);
    uint8_t* ring = smem + L.ring;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
    uint64_t* empty = full + kSStagesMax;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kSStagesMax);
    __shared__ int touched_ids[256];  // touched experts in id order (E <= 256)
    __shared__ int n_touched;
    float* xch = reinterpret_cast<float*>(smem + L.xch);
    uint8_t* xs = smem + L.rows;
    float* cs = reinterpret_cast<float*>(smem + L.sums);

    if (tid == 0) {
        for (int s = 0; s < stages; ++s) {
            sbar_init(s_addr(&full[s]), 1);
            sbar_init(s_addr(&empty[s]), kSCons / 2);
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    pdl_trigger();
    pdl_wait();  // the segment offsets, row map and activations come from earlier kernels
    // touched experts, in id order (one warp)
    if (warp == 0) {
        int base = 0;
        for (int e0 = 0; e0 < a.E; e0 += 32) {
            const int e = e0 + lane;
            const bool t = e < a.E && a.offsets[e + 1] > a.offsets[e];
            const uint32_t m = __ballot_sync(0xffffffffu, t);
            if (t) touched_ids[base + __popc(m & ((1u << lane) - 1u))] = e;
            base += __popc(m);
        }
        if (lane == 0) n_touched = base;
    }
    __syncthreads();
    const int n_items = n_touched * nrb * a.splits;
    const int i_lo = int((int64_t(blockIdx.x) * n_items) / gridDim.x);
    const int i_hi = int((int64_t(blockIdx.x + 1) * n_items) / gridDim.x);

    if (warp == kSCons) {
        // ---------------------------------------------------------- producer
        int st = 0;
        uint32_t ph = 0;
        bool ok = true;
        for (int i = i_lo; ok && i < i_hi; ++i) {
            const SItem it = stream_item(i, nrb, a.splits, touched_ids);
            const int M = a.offsets[it.e + 1] - a.offsets[it.e];
            int64_t g_lo, g_hi;
            split_range(ngr, a.splits, it.split, gpb, g_lo, g_hi);
            const uint8_t* base = a.W + ((int64_t(it.e) * nrb + it.rb) * ngr) * int64_t(kSSlab);
            for (int p0 = 0; ok && p0 < M; p0 += ROWS) {
                for (int64_t g = g_lo; g < g_hi; ++g) {
                    if (!sbar_wait(s_addr(&empty[st]), ph ^ 1u, abort_flag, status)) { ok = false; break; }
                    if (lane == 0) {
                        sbar_expect(s_addr(&full[st]), kSSlab);
                        bulk_slab(s_addr(ring + st * kSSlab), base + g * kSSlab, s_addr(&full[st]));
                    }
                    __syncwarp();
                    if (++st == stages) { st = 0; ph ^= 1u; }
                }
            }
        }
        return;  // the consumers never wait on the producer at a barrier
    }

    // ---------------------------------------------------------------- consumers
    const int tile = warp & 7, par = warp >> 3;
    const int r0 = lane >> 2, c = lane & 3;
    const __nv_bfloat16* act = (const __nv_bfloat16*)a.act;
    int st = 0;
    uint32_t ph = 0;
    int staged_e = -1, staged_split = -1, staged_p0 = -1;
    for (int i = i_lo; i < i_hi; ++i) {
        const SItem it = stream_item(i, nrb, a.splits, touched_ids);
        const int64_t seg0 = a.offsets[it.e];
        const int M = a.offsets[it.e + 1] - int(seg0);
        int64_t g_lo, g_hi;
        split_range(ngr, a.splits, it.split, gpb, g_lo, g_hi);
        const int ng = int(g_hi - g_lo);
        const int kr = ng * KG;
        const int rs = int(stream_row_bytes(kr));
        const int64_t rt = int64_t(it.rb) * kTilesPerBlock + tile;
        const bool active = rt < nrt;
        const int64_t sb0 = ((int64_t(it.e) * nrb + it.rb) * nsb * kTilesPerBlock + tile) * 16 + 2 * r0;
        const void* sbase = SF32 ? (const void*)((const float*)a.S + sb0) : (const void*)((const __nv_bfloat16*)a.S + sb0);
        float s0 = 1.0f, s1 = 1.0f;  // per-column scales
        if (SMODE == 0 && active) ScaleRaw<SF32>::load(sbase, 0).get(s0, s1);

        for (int p0 = 0; p0 < M; p0 += ROWS) {
            if (it.e != staged_e || it.split != staged_split || p0 != staged_p0) {
                // rows p0 .. p0 + ROWS - 1 of the expert's segment (clamped) and
                // their sums, per k-group (block scales) or over the range
                consumers_sync();  // every consumer is done with the previous rows
                for (int row = warp; row < ROWS; row += kSCons) {
                    const int tok = min(p0 + row, M - 1);
                    const int64_t srow = a.rowmap ? a.rowmap[seg0 + tok] : seg0 + tok;
                    const __nv_bfloat16* src = act + srow * a.K + g_lo * KG;
                    uint8_t* dst = xs + row * rs;
                    for (int ch = lane; ch < kr / 8; ch += 32) cp_async16(dst + ch * 16, src + ch * 8);
                }
                cp_async_wait_all();
                consumers_sync();
                if (FOLD && SMODE == 1) {
                    // one thread per (k-group, row): fp32 sum in k order
                    for (int q = tid; q < ng * ROWS; q += kSCons * 32) {
                        const int g = q / ROWS, row = q - g * ROWS;
                        const uint4* src = reinterpret_cast<const uint4*>(xs + row * rs + g * KG * 2);
                        float sum = 0.0f;
#pragma unroll
                        for (int v8 = 0; v8 < KG / 8; ++v8) {
                            const uint4 v = src[v8];
                            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                            for (int h = 0; h < 4; ++h) {
                                sum += __uint_as_float(u[h] << 16);
                                sum += __uint_as_float(u[h] & 0xFFFF0000u);
                            }
                        }
                        cs[q] = sum;
                    }
                    consumers_sync();
                } else if (FOLD) {
                    // one warp per row: strided partial sums, then a fixed shuffle tree
                    for (int row = warp; row < ROWS; row += kSCons) {
                        const uint4* src = reinterpret_cast<const uint4*>(xs + row * rs);
                        float sum = 0.0f;
                        for (int q = lane; q < kr / 8; q += 32) {
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
                    consumers_sync();
                }
                staged_e = it.e;
                staged_split = it.split;
                staged_p0 = p0;
            }

            float acc[NT][4];
#pragma unroll
            for (int n = 0; n < NT; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.0f;
            const uint8_t* xp = xs + r0 * rs + 8 * c;
            // the scale pair of this warp's next k-group, one group ahead
            auto sload = [&](int g) -> ScaleRaw<SF32> {
                return ScaleRaw<SF32>::load(sbase, ((int(g_lo) + g) >> lg_gpb) * 128);
            };
            ScaleRaw<SF32> s_next{};
            if (SMODE == 1 && active && par < ng) s_next = sload(par);

            for (int g = 0; g < ng; ++g) {
                if ((g & 1) == par) {
                    if (!*abort_flag && sbar_wait(s_addr(&full[st]), ph, abort_flag, status)) {
                        const uint4 w = *reinterpret_cast<const uint4*>(ring + st * kSSlab + (tile * 32 + lane) * 16);
                        const uint8_t* xg = xp + g * KG * 2;
                        uint2 xa[NT][KSTEPS];
#pragma unroll
                        for (int n = 0; n < NT; ++n)
#pragma unroll
                            for (int j = 0; j < KSTEPS; ++j)
                                xa[n][j] = *reinterpret_cast<const uint2*>(xg + n * 8 * rs + j * 32);
                        float2 fs[NT];
                        if (FOLD && SMODE == 1)
#pragma unroll
                            for (int n = 0; n < NT; ++n) fs[n] = *reinterpret_cast<const float2*>(cs + g * ROWS + 8 * n + 2 * c);
                        const ScaleRaw<SF32> sc = s_next;
                        if (SMODE == 1 && active && g + 2 < ng) s_next = sload(g + 2);
                        __syncwarp();
                        if (lane == 0) sbar_arrive(s_addr(&empty[st]));  // the slab is in registers now
                        const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
                        float blk[NT][4];
#pragma unroll
                        for (int j = 0; j < KSTEPS; ++j) {
                            uint32_t A[4];
                            if (BITS == 4) {
                                constexpr uint32_t kMask = 0x000F000Fu, kMagic = 0x43004300u;
                                A[0] = (wv[j] & kMask) | kMagic;
                                A[1] = ((wv[j] >> 4) & kMask) | kMagic;
                                A[2] = ((wv[j] >> 8) & kMask) | kMagic;
                                A[3] = ((wv[j] >> 12) & kMask) | kMagic;
                            } else {
                                const uint32_t lo = wv[2 * j], hi = wv[2 * j + 1];
                                float f[8];
#pragma unroll
                                for (int m = 0; m < 4; ++m) {
                                    f[m] = byte_centered(lo, m);
                                    f[4 + m] = byte_centered(hi, m);
                                }
#pragma unroll
                                for (int q = 0; q < 4; ++q) A[q] = pack_bf2(f[2 * q], f[2 * q + 1]);
                            }
#pragma unroll
                            for (int n = 0; n < NT; ++n) {
                                if (SMODE == 1) {
                                    if (j == 0)
                                        mma_bf16_zero(blk[n], A, xa[n][j].x, xa[n][j].y);
                                    else
                                        mma_bf16(blk[n], A, xa[n][j].x, xa[n][j].y);
                                } else {
                                    mma_bf16(acc[n], A, xa[n][j].x, xa[n][j].y);
                                }
                            }
                        }
                        if (SMODE == 1) {
                            float sa, sb;
                            sc.get(sa, sb);
#pragma unroll
                            for (int n = 0; n < NT; ++n) {
                                if (FOLD) {
                                    blk[n][0] = fmaf(-kFold, fs[n].x, blk[n][0]);
                                    blk[n][1] = fmaf(-kFold, fs[n].y, blk[n][1]);
                                    blk[n][2] = fmaf(-kFold, fs[n].x, blk[n][2]);
                                    blk[n][3] = fmaf(-kFold, fs[n].y, blk[n][3]);
                                }
                                acc[n][0] = fmaf(sa, blk[n][0], acc[n][0]);
                                acc[n][1] = fmaf(sa, blk[n][1], acc[n][1]);
                                acc[n][2] = fmaf(sb, blk[n][2], acc[n][2]);
                                acc[n][3] = fmaf(sb, blk[n][3], acc[n][3]);
                            }
                        }
                    }
                }
                if (++st == stages) { st = 0; ph ^= 1u; }
            }

            // the odd-group warp of each tile hands its half to the even one,
            // which finishes the fold (per-column mode), scales and stores
            float* mine = xch + ((tile * 32 + lane) * NT) * 4;
            if (par == 1)
#pragma unroll
                for (int n = 0; n < NT; ++n)
#pragma unroll
                    for (int q = 0; q < 4; ++q) mine[n * 4 + q] = acc[n][q];
            consumers_sync();
            if (par == 0 && active && !*abort_flag) {
#pragma unroll
                for (int n = 0; n < NT; ++n) {
                    float v[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) v[q] = acc[n][q] + mine[n * 4 + q];
                    if (SMODE == 0) {
                        if (FOLD) {
                            const float2 t = *reinterpret_cast<const float2*>(cs + 8 * n + 2 * c);
                            v[0] = fmaf(-kFold, t.x, v[0]);
                            v[1] = fmaf(-kFold, t.y, v[1]);
                            v[2] = fmaf(-kFold, t.x, v[2]);
                            v[3] = fmaf(-kFold, t.y, v[3]);
                        }
                        v[0] *= s0;
                        v[1] *= s0;
                        v[2] *= s1;
                        v[3] *= s1;
                    }
                    epilogue(a, it.e, rt, r0, c, seg0, M, p0 + 8 * n, v, it.split, true);
                }
            }
            consumers_sync();  // the exchange slots are read before the next item writes them
        }
    }
}

template <int BITS, int SMODE, bool SF32, int NT>
cudaError_t launch_t(const FfnArgs& a, int32_t* status, int grid, size_t smem, int stages, cudaStream_t st) {
    return launch_kernel(ffn_stream_kernel<BITS, SMODE, SF32, NT>, dim3(unsigned(grid)), dim3(kSThreads), smem, st,
                         a.pdl != 0, a, status, stages);
}

template <int BITS, int SMODE, bool SF32, int NT>
cudaError_t prepare_t() {
    return cudaFuncSetAttribute(ffn_stream_kernel<BITS, SMODE, SF32, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                int(kStreamSmemLimit));
}

template <int BITS, int SMODE, bool SF32>
cudaError_t launch_nt(const FfnArgs& a, int32_t* status, int grid, size_t smem, int stages, cudaStream_t st) {
    return a.nt == 1 ? launch_t<BITS, SMODE, SF32, 1>(a, status, grid, smem, stages, st)
                     : launch_t<BITS, SMODE, SF32, 2>(a, status, grid, smem, stages, st);
}

template <int BITS, int SMODE>
cudaError_t launch_sf(const FfnArgs& a, int32_t* status, int grid, size_t smem, int stages, cudaStream_t st) {
    return a.scale_bf16 ? launch_nt<BITS, SMODE, false>(a, status, grid, smem, stages, st)
                        : launch_nt<BITS, SMODE, true>(a, status, grid, smem, stages, st);
}

template <int BITS, int SMODE>
cudaError_t prepare_sf() {
    cudaError_t e = prepare_t<BITS, SMODE, false, 1>();
    if (e == cudaSuccess) e = prepare_t<BITS, SMODE, false, 2>();
    if (e == cudaSuccess) e = prepare_t<BITS, SMODE, true, 1>();
    if (e == cudaSuccess) e = prepare_t<BITS, SMODE, true, 2>();
    return e;
}

}  // namespace

bool stream_supports(int bits, int block_size, int fp4, int nt) {
    return !fp4 && nt <= 2 && (block_size == 0 || block_size >= kgroup_of(bits));
}

int64_t stream_smem_bytes(int64_t K, int bits, int block_size, int splits, int nt, int* stages_out) {
    const int kg = kgroup_of(bits);
    const int64_t ngr = K / kg;
    const int64_t gpb = block_size >= kg ? block_size / kg : 1;
    const int64_t nblk = (ngr + gpb - 1) / gpb;
    const int64_t per = (nblk + splits - 1) / splits;
    const int64_t ng = std::min<int64_t>(ngr, per * gpb);
    // as many ring slabs as fit (4 .. 16), the rest of the CTA's memory fixed
    const StreamLayout base = stream_layout(ng * kg, int(ng), nt, 0);
    int stages = int(std::min<int64_t>(kSStagesMax, (int64_t(kStreamSmemLimit) - base.total) / kSSlab));
    if (stages_out) *stages_out = stages;
    if (stages < 4) return int64_t(kStreamSmemLimit) + 1;
    return stream_layout(ng * kg, int(ng), nt, stages).total;
}

cudaError_t prepare_ffn_stream() {
    cudaError_t e = prepare_sf<4, 0>();
    if (e == cudaSuccess) e = prepare_sf<4, 1>();
    if (e == cudaSuccess) e = prepare_sf<8, 0>();
    if (e == cudaSuccess) e = prepare_sf<8, 1>();
    return e;
}

cudaError_t launch_ffn_stream(const FfnArgs& a, int32_t* status, cudaStream_t st) {
    if (!stream_supports(a.bits, a.block_size, a.fp4, a.nt) || a.E > 256) return cudaErrorInvalidConfiguration;
    int stages = 0;
    const int64_t smem = stream_smem_bytes(a.K, a.bits, a.block_size, a.splits, a.nt, &stages);
    if (smem > int64_t(kStreamSmemLimit)) return cudaErrorInvalidConfiguration;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int smode = a.block_size == 0 ? 0 : 1;
    if (a.bits == 4)
        return smode == 0 ? launch_sf<4, 0>(a, status, sms, size_t(smem), stages, st)
                          : launch_sf<4, 1>(a, status, sms, size_t(smem), stages, st);
    return smode == 0 ? launch_sf<8, 0>(a, status, sms, size_t(smem), stages, st)
                      : launch_sf<8, 1>(a, status, sms, size_t(smem), stages, st);
}

}  // namespace qmoe
