// ffn_tc.cu -- expert FFN layers on the 5th-generation tensor cores
// (tcgen05.mma with TMEM accumulators), sm_100a.
//
// Each linear is y = x @ dequant(W).T + b ("QLinearWoQ" page, class summary)
// over the rows routed to one expert; the packed weights are decoded one
// 128 x 64 tile at a time inside the GEMM mainloop and never written out
// dense in global memory ("ClikaRT::nn::QMoEWoQ", class description: each
// expert weight decodes one block at a time inside the GEMM dot). FC1 applies
// the QMoE page's gated activation in its epilogue.
//
// Operand roles ("swap AB"): the MMA's M dimension is 128 weight rows, its N
// dimension the routed tokens of one expert (a multiple of 16, up to 128), so
// a small expert segment wastes no tensor work on padding rows.
//
// Warp roles of one persistent CTA (576 threads, one CTA per SM):
//   warps 0-7   dequantise: packed codes (shared) -> bf16 A tile written
//               straight into tensor memory (tcgen05.st), one 16-row tile per
//               warp; the A operand never touches shared memory
//   warp 8      producer: one bulk copy of the packed 128 x 64 tile (4 KB
//               int4, 8 KB int8), one of its scales, and 64-row TMA boxes of
//               the activations (bf16, 128-byte swizzle), as many as the tile
//               has rows
//   warp 9      allocates TMEM and issues tcgen05.mma (A from TMEM, B from
//               shared memory) from one thread
//   warps 10-17 epilogue: TMEM -> registers (tcgen05.ld), scale / bias /
//               activation, global stores; two warps per TMEM lane quarter
// Stages cycle through an S-deep ring guarded by mbarriers (full: copies
// landed; deq: A tile written to TMEM; empty: the MMAs reading the stage are
// done); two TMEM accumulators let the epilogue of one work item overlap the
// mainloop of the next. Every wait is bounded: after about two seconds the
// kernel records QMOE_TIMEOUT in the workspace status word, every role
// leaves its loop, and the CTA frees its TMEM and exits.
//
// The packed layout puts lane (r0 = L/4, c = L%4) of a 16-row tile on rows r0
// and r0 + 8 and k = 16j + 4c + {0..3}: after decoding, its registers are
// exactly the 16x256b tensor-memory store fragment of k-step j.
//
// Scales: a K-block scale is multiplied into the decoded weight (one bf16
// rounding of (q - z) * s); per-column scales (block_size 0) leave exact
// integer weights in the MMA and are applied in fp32 in the epilogue.
#include <cuda.h>

#include "qmoe_internal.cuh"

namespace qmoe {
namespace {

constexpr int kDeqWarps = 8;
constexpr int kWarpProd = 8;
constexpr int kWarpMma = 9;
constexpr int kWarpEpi0 = 10;
constexpr int kEpiWarps = 8;
constexpr int kTcThreads = (kWarpEpi0 + kEpiWarps) * 32;  // 576
constexpr int kBK = 64;                                    // k per stage
constexpr int kAStageCols = kBK / 2;                       // TMEM columns of one A tile
constexpr int kScaleBytesMax = 4 * kTilesPerBlock * 16 * 4;  // 4 blocks of fp32 pairs
constexpr uint64_t kTimeoutNs = 2000000000ull;

struct TcArgs {
    const uint8_t* W;
    const void* S;
    const float* bias;       // FC1, packed row order, or nullptr
    const int32_t* offsets;  // [E + 1]
    void* out;               // FC1: h [R, I] bf16; FC2: partials [splits, R, N] fp32
    int32_t* status;         // workspace status word
    int64_t N, K, R;
    int E, block_size, gated, is_fc1, act_type;
    float alpha, beta, limit;
    int splits, scale_bf16, bn;
    int ring, stage_bytes;   // streaming decode: packed-ring depth and slot size
};

// ------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return uint32_t(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        "selp.b32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t now_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Bounded wait on a phase parity. Returns false (after raising the CTA's
// abort flag and the workspace status) when the wait gives up or another role
// already aborted.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          int32_t* status) {
    if (mbar_try(bar, parity)) return true;
    const uint64_t t0 = now_ns();
    for (uint32_t spin = 1;; ++spin) {
        if (mbar_try(bar, parity)) return true;
        if ((spin & 255u) == 0u) {
            if (*abort_flag) return false;
            if (now_ns() - t0 > kTimeoutNs) {
                *abort_flag = 1;
                atomicExch(status, int32_t(QMOE_TIMEOUT));
                return false;
            }
        }
    }
}

// Wait by a whole warp: every lane polls, and the warp continues only if all
// lanes saw the phase complete (a timeout in any lane stops the whole warp).
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          int32_t* status) {
    const bool ok = mbar_wait(bar, parity, abort_flag, status);
    return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void tma_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                       uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, "
        "{%2, %3}], [%4];" ::"r"(dst),
        "l"(map), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row atoms of
// 1024 bytes stacked along M/N (stride 1024), version 1 for sm_100.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr) {
    uint64_t d = uint64_t((saddr >> 4) & 0x3FFFu);
    d |= uint64_t(1) << 16;             // leading offset: unused for swizzled K-major
    d |= uint64_t(1024 >> 4) << 32;     // stride offset between 8-row atoms
    d |= uint64_t(1) << 46;             // descriptor version
    d |= uint64_t(2) << 61;             // 128-byte swizzle
    return d;
}

// Instruction descriptor: kind::f16, bf16 A and B (K-major), fp32 D, M = 128.
__device__ __forceinline__ uint32_t idesc_bf16(int n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(n >> 3) << 17) | (uint32_t(128 >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16_ss(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st16x256_x4(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.16x256b.x4.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
        "%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

__device__ __forceinline__ void tmem_st16x256_x2(uint32_t taddr, const uint32_t (&r)[8]) {
    asm volatile(
        "tcgen05.st.sync.aligned.16x256b.x2.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
        : "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// MMA with A read from tensor memory (128 lanes = rows, 2 bf16 per column).
__device__ __forceinline__ void mma_bf16_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}" ::"r"(tmem_d),
        "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// Single-issuer instructions from a converged warp: the whole warp runs the
// issuing loop (so its control flow and operands stay warp-uniform) and the
// instruction itself is predicated on one elected lane, with no branch.
__device__ __forceinline__ uint32_t elect_one() {
    uint32_t e;
    asm volatile("{\n.reg .pred p;\nelect.sync _|p, 0xffffffff;\nselp.b32 %0, 1, 0, p;\n}" : "=r"(e));
    return e;
}

__device__ __forceinline__ void mma_bf16_ts_e(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                              uint32_t accumulate, uint32_t e) {
    asm volatile(
        "{\n.reg .pred p, q;\nsetp.ne.b32 p, %4, 0;\nsetp.ne.b32 q, %5, 0;\n"
        "@q tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}" ::"r"(tmem_d),
        "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(e));
}

__device__ __forceinline__ void mma_commit_e(uint32_t bar, uint32_t e) {
    asm volatile(
        "{\n.reg .pred q;\nsetp.ne.b32 q, %1, 0;\n"
        "@q tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n}" ::"r"(bar),
        "r"(e)
        : "memory");
}

__device__ __forceinline__ void mbar_expect_tx_e(uint32_t bar, uint32_t bytes, uint32_t e) {
    asm volatile(
        "{\n.reg .pred q;\nsetp.ne.b32 q, %2, 0;\n"
        "@q mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n}" ::"r"(bar),
        "r"(bytes), "r"(e)
        : "memory");
}

__device__ __forceinline__ void bulk_g2s_e(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar,
                                           uint32_t e) {
    asm volatile(
        "{\n.reg .pred q;\nsetp.ne.b32 q, %4, 0;\n"
        "@q cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n}" ::"r"(
            dst),
        "l"(src), "r"(bytes), "r"(bar), "r"(e)
        : "memory");
}

__device__ __forceinline__ void tma_3d_e(uint32_t dst, const CUtensorMap* map, int x, int y, int z,
                                         uint32_t bar, uint32_t e) {
    asm volatile(
        "{\n.reg .pred q;\nsetp.ne.b32 q, %6, 0;\n"
        "@q cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, "
        "{%2, %3, %4}], [%5];\n}" ::"r"(dst),
        "l"(map), "r"(x), "r"(y), "r"(z), "r"(bar), "r"(e)
        : "memory");
}

__device__ __forceinline__ void tma_2d_e(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar,
                                         uint32_t e) {
    asm volatile(
        "{\n.reg .pred q;\nsetp.ne.b32 q, %5, 0;\n"
        "@q cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, "
        "{%2, %3}], [%4];\n}" ::"r"(dst),
        "l"(map), "r"(x), "r"(y), "r"(bar), "r"(e)
        : "memory");
}

// --------------------------------------------------------------- arithmetic
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
__device__ __forceinline__ uint32_t bf2_bcast(float s) {
    __nv_bfloat162 r = __float2bfloat162_rn(s);
    return *reinterpret_cast<uint32_t*>(&r);
}

// fast sigmoid: the result is rounded to bf16 right after
__device__ __forceinline__ float sigmoidf_(float v) { return __fdividef(1.0f, 1.0f + __expf(-v)); }
__device__ __forceinline__ float act_plain(int t, float a) {
    switch (t) {
        case QMOE_ACT_RELU: return fmaxf(a, 0.0f);
        case QMOE_ACT_GELU: return 0.5f * a * (1.0f + erff(a * 0.70710678118654752f));
        case QMOE_ACT_SILU: return a * sigmoidf_(a);
        default: return a;
    }
}
__device__ __forceinline__ float act_gated(int t, float g, float u, float alpha, float beta,
                                           float limit) {
    if (t == QMOE_ACT_SWIGLU) {
        g = fminf(g, limit);
        u = fminf(fmaxf(u, -limit), limit);
        return (u + beta) * g * sigmoidf_(alpha * g);
    }
    return act_plain(t, g) * u;
}

// ------------------------------------------------------------ work items
struct Item {
    int e, rb, tt, split;
    int64_t seg0;
    int M;      // rows routed to the expert
    int rows;   // rows of this token tile
    int ks_lo, ks_hi;
};

// Items are ordered expert, row block, token tile, split, so CTAs working on
// neighbouring items share weight blocks in L2.
__device__ __forceinline__ Item item_at(int i, const int* prefix, const TcArgs& a, int nrb, int nks) {
    int lo = 0, hi = a.E;  // largest e with prefix[e] <= i
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (prefix[mid] <= i) lo = mid; else hi = mid;
    }
    Item it;
    it.e = lo;
    it.seg0 = a.offsets[lo];
    it.M = a.offsets[lo + 1] - int(it.seg0);
    const int ntt = (it.M + a.bn - 1) / a.bn;
    int rem = i - prefix[lo];
    const int per_rb = ntt * a.splits;
    it.rb = rem / per_rb;
    rem -= it.rb * per_rb;
    it.tt = rem / a.splits;
    it.split = rem - it.tt * a.splits;
    it.rows = min(a.bn, it.M - it.tt * a.bn);
    it.ks_lo = int((int64_t(it.split) * nks) / a.splits);
    it.ks_hi = int((int64_t(it.split + 1) * nks) / a.splits);
    return it;
}

template <int BITS, bool PERCOL, int BNMAX, int STAGES>
struct TcCfg {
    static constexpr int kBoxRows = BNMAX < 64 ? BNMAX : 64;       // rows of one activation TMA box
    static constexpr int kPacked = kBlockRows * kBK * BITS / 8;    // 4 KB or 8 KB
    static constexpr int kB = BNMAX * 128;                         // activation tile
    static constexpr int kStage = kB + kPacked + kScaleBytesMax;   // multiple of 1024
    static constexpr int kACol0 = 2 * BNMAX;                       // A tiles after the accumulators
    static constexpr int kTmemCols = 512;
    static_assert(kACol0 + STAGES * kAStageCols <= kTmemCols, "TMEM budget");
    static constexpr int kBarOff = STAGES * kStage;
    // barriers, prefix table, alignment slack; at least 120 KB so one CTA per SM
    static constexpr int kSmemUse = kBarOff + 1024 + 4 * 260 + 1024;
    static constexpr int kSmem = kSmemUse > 120 * 1024 ? kSmemUse : 120 * 1024;
};

template <int BITS, bool PERCOL, int BNMAX, int STAGES>
__global__ void __launch_bounds__(kTcThreads, 1)
    ffn_tc_kernel(const __grid_constant__ CUtensorMap bmap, const TcArgs a) {
    using C = TcCfg<BITS, PERCOL, BNMAX, STAGES>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    uint8_t* bar_area = smem + C::kBarOff;
    uint64_t* full = reinterpret_cast<uint64_t*>(bar_area);
    uint64_t* deq = full + STAGES;
    uint64_t* empty = deq + STAGES;
    uint64_t* accf = empty + STAGES;
    uint64_t* acce = accf + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acce + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* prefix = reinterpret_cast<int*>(tmem_slot + 4);  // [E + 1]

    const int nrb = int(padded_rows(a.N) / kBlockRows);
    const int nks = int(a.K / kBK);

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&deq[s]), kDeqWarps);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&accf[b]), 1);
            mbar_init(smem_u32(&acce[b]), kEpiWarps);
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {  // item counts per expert, exclusive prefix
        int carry = 0;
        for (int e0 = 0; e0 < a.E; e0 += 32) {
            const int e = e0 + lane;
            int v = 0;
            if (e < a.E) {
                const int M = a.offsets[e + 1] - a.offsets[e];
                v = ((M + a.bn - 1) / a.bn) * nrb * a.splits;
            }
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += n;
            }
            if (e < a.E) prefix[e] = carry + incl - v;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) prefix[a.E] = carry;
    }
    if (warp == kWarpMma) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(C::kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int total = prefix[a.E];
    const int nsb = a.block_size > 0 ? int(a.K / a.block_size) : 1;
    const int ssz = a.scale_bf16 ? 2 : 4;
    // scale blocks covered by one 64-k stage, and the stage's scale bytes
    const int sblk = PERCOL ? 0 : (a.block_size >= kBK ? 1 : kBK / a.block_size);
    const uint32_t sbytes = uint32_t(sblk * kTilesPerBlock * 16 * ssz);

    if (warp == kWarpProd) {
        // ------------------------------------------------------- producer
        {
            const uint32_t e = elect_one();
            int st = 0;
            uint32_t ph = 0;
            bool ok = true;
            const int ngr = int(a.K / kgroup_of(BITS));
            for (int i = blockIdx.x; ok && i < total; i += gridDim.x) {
                const Item it = item_at(i, prefix, a, nrb, nks);
                const int nbox = (it.rows + C::kBoxRows - 1) / C::kBoxRows;
                const uint32_t bytes = uint32_t(C::kPacked + nbox * C::kBoxRows * 128) + sbytes;
                for (int ks = it.ks_lo; ks < it.ks_hi; ++ks) {
                    if (!warp_wait(smem_u32(&empty[st]), ph ^ 1u, abort_flag, a.status)) { ok = false; break; }
                    uint8_t* sb = smem + st * C::kStage;
                    const uint32_t fb = smem_u32(&full[st]);
                    mbar_expect_tx_e(fb, bytes, e);
                    const int g = ks * (kBK / kgroup_of(BITS));  // first k-group of the stage
                    const uint8_t* src =
                        a.W + ((int64_t(it.e) * nrb + it.rb) * ngr + g) * int64_t(kTilesPerBlock) * kUnitBytes;
                    bulk_g2s_e(smem_u32(sb + C::kB), src, C::kPacked, fb, e);
                    if (!PERCOL) {
                        const int b0 = (ks * kBK) / a.block_size;
                        const int64_t sidx = ((int64_t(it.e) * nrb + it.rb) * nsb + b0) * kTilesPerBlock * 16;
                        const uint8_t* ssrc = reinterpret_cast<const uint8_t*>(a.S) + sidx * ssz;
                        bulk_g2s_e(smem_u32(sb + C::kB + C::kPacked), ssrc, sbytes, fb, e);
                    }
                    const int y0 = int(it.seg0) + it.tt * a.bn;
                    for (int b = 0; b < nbox; ++b)
                        tma_2d_e(smem_u32(sb + b * C::kBoxRows * 128), &bmap, ks * kBK, y0 + b * C::kBoxRows, fb, e);
                    if (++st == STAGES) { st = 0; ph ^= 1u; }
                }
            }
        }
    } else if (warp == kWarpMma) {
        // ------------------------------------------------------- MMA issuer
        {
            const uint32_t e = elect_one();
            int st = 0, acc = 0;
            uint32_t ph = 0, aph = 0;
            bool ok = true;
            for (int i = blockIdx.x; ok && i < total; i += gridDim.x) {
                const Item it = item_at(i, prefix, a, nrb, nks);
                const int n = ((it.rows + 15) / 16) * 16;
                const uint32_t idesc = idesc_bf16(n);
                if (!warp_wait(smem_u32(&acce[acc]), aph ^ 1u, abort_flag, a.status)) break;
                tc_fence_after();
                const uint32_t d = tmem + uint32_t(acc * BNMAX);
                for (int ks = it.ks_lo; ks < it.ks_hi; ++ks) {
                    if (!warp_wait(smem_u32(&deq[st]), ph, abort_flag, a.status) ||
                        !warp_wait(smem_u32(&full[st]), ph, abort_flag, a.status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t at = tmem + uint32_t(C::kACol0 + st * kAStageCols);
                    const uint64_t bd = desc_sw128(smem_u32(smem + st * C::kStage));
                    const uint32_t acc0 = ks > it.ks_lo ? 1u : 0u;
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)  // 16 k per MMA: 8 A columns, 32 B of B
                        mma_bf16_ts_e(d, at + uint32_t(8 * kk), bd + uint64_t(2 * kk), idesc, kk > 0 ? 1u : acc0, e);
                    mma_commit_e(smem_u32(&empty[st]), e);
                    if (++st == STAGES) { st = 0; ph ^= 1u; }
                }
                if (!ok) break;
                mma_commit_e(smem_u32(&accf[acc]), e);
                if (++acc == 2) { acc = 0; aph ^= 1u; }
            }
        }
    } else if (warp < kDeqWarps) {
        // ------------------------------------------------------- dequantise
        // warp w writes row tile t = 2*(w%4) + w/4 (TMEM lanes 16t..16t+15,
        // inside the lane quarter w%4 it may access)
        const int tile = 2 * (warp & 3) + (warp >> 2);
        const int r0 = lane >> 2, c = lane & 3;
        const uint32_t lane_addr = uint32_t(16 * tile) << 16;
        int st = 0;
        uint32_t ph = 0;
        bool ok = true;
        const uint32_t kMask = 0x000F000Fu, kMagic = 0x43004300u, kBias4 = 0x43084308u;
        for (int i = blockIdx.x; ok && i < total; i += gridDim.x) {
            const Item it = item_at(i, prefix, a, nrb, nks);
            for (int ks = it.ks_lo; ks < it.ks_hi; ++ks) {
                if (!warp_wait(smem_u32(&full[st]), ph, abort_flag, a.status)) { ok = false; break; }
                const uint8_t* sb = smem + st * C::kStage;
                const uint8_t* pk = sb + C::kB;
                const uint8_t* sc = pk + C::kPacked;
                const uint32_t at = tmem + lane_addr + uint32_t(C::kACol0 + st * kAStageCols);
                constexpr int GROUPS = kBK / kgroup_of(BITS);  // 1 (int4) or 2 (int8)
#pragma unroll
                for (int gg = 0; gg < GROUPS; ++gg) {
                    const uint4 w = *reinterpret_cast<const uint4*>(pk + ((gg * kTilesPerBlock + tile) * 32 + lane) * 16);
                    const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
                    constexpr int KSTEPS = kgroup_of(BITS) / 16;
                    uint32_t r[4 * KSTEPS];
#pragma unroll
                    for (int j = 0; j < KSTEPS; ++j) {
                        uint32_t A[4];  // (r0, k 0-1), (r0+8, k 0-1), (r0, k 2-3), (r0+8, k 2-3)
                        if (BITS == 4) {
                            A[0] = bf2_sub((wv[j] & kMask) | kMagic, kBias4);
                            A[1] = bf2_sub(((wv[j] >> 4) & kMask) | kMagic, kBias4);
                            A[2] = bf2_sub(((wv[j] >> 8) & kMask) | kMagic, kBias4);
                            A[3] = bf2_sub(((wv[j] >> 12) & kMask) | kMagic, kBias4);
                        } else {
                            // byte b holds q - 128 = (b & 127) - (b < 128 ? 128 : 0): OR the
                            // low 7 bits into bf16 128.0 and subtract 256.0 or 128.0 (0x4380
                            // with its exponent bit flipped by the byte's top bit), exactly
#pragma unroll
                            for (int qq = 0; qq < 4; ++qq) {
                                const uint32_t word = wv[2 * j + (qq >> 1)];
                                const uint32_t pr = __byte_perm(word, 0u, (qq & 1) ? 0x4342u : 0x4140u);
                                const uint32_t lo = (pr & 0x007F007Fu) | 0x43004300u;
                                const uint32_t hi = (pr & 0x00800080u) ^ 0x43804380u;
                                A[qq] = bf2_sub(lo, hi);
                            }
                        }
                        if (!PERCOL) {
                            // scale block of this k-step (k = 64*ks + 32*gg + 16j + 4c + ...)
                            const int kl = 32 * gg * (BITS == 8) + 16 * j + 4 * c;
                            const int blk = a.block_size >= kBK ? 0 : kl / a.block_size;
                            const int si = (blk * kTilesPerBlock + tile) * 16 + 2 * r0;
                            float sa, sbv;
                            if (a.scale_bf16) {
                                const uint32_t raw = *reinterpret_cast<const uint32_t*>(sc + si * 2);
                                sa = __uint_as_float(raw << 16);
                                sbv = __uint_as_float(raw & 0xFFFF0000u);
                            } else {
                                const float2 f = *reinterpret_cast<const float2*>(sc + si * 4);
                                sa = f.x;
                                sbv = f.y;
                            }
                            const uint32_t sa2 = bf2_bcast(sa), sb2 = bf2_bcast(sbv);
                            A[0] = bf2_mul(A[0], sa2);
                            A[2] = bf2_mul(A[2], sa2);
                            A[1] = bf2_mul(A[1], sb2);
                            A[3] = bf2_mul(A[3], sb2);
                        }
                        // 16x256b fragment: (r0, col 2c), (r0, col 2c+1), (r0+8, col 2c), (r0+8, col 2c+1)
                        r[4 * j + 0] = A[0];
                        r[4 * j + 1] = A[2];
                        r[4 * j + 2] = A[1];
                        r[4 * j + 3] = A[3];
                    }
                    if (BITS == 4) {
                        tmem_st16x256_x4(at, *reinterpret_cast<const uint32_t(*)[16]>(r));
                    } else {
                        tmem_st16x256_x2(at + uint32_t(16 * gg), *reinterpret_cast<const uint32_t(*)[8]>(r));
                    }
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&deq[st]));
                if (++st == STAGES) { st = 0; ph ^= 1u; }
            }
        }
    } else if (warp >= kWarpEpi0) {
        // ------------------------------------------------------- epilogue
        const int qd = warp & 3;                        // TMEM lane quarter this warp may read
        const int half = (warp - kWarpEpi0) >> 2;       // which 16-column chunks it takes
        const int row = qd * 32 + lane;
        int acc = 0;
        uint32_t aph = 0;
        for (int i = blockIdx.x; i < total; i += gridDim.x) {
            const Item it = item_at(i, prefix, a, nrb, nks);
            if (!warp_wait(smem_u32(&accf[acc]), aph, abort_flag, a.status)) break;
            tc_fence_after();
            const int64_t prow = int64_t(it.rb) * kBlockRows + row;  // packed row in the expert
            const bool valid = prow < a.N;
            float s = 1.0f;
            if (PERCOL && valid) {
                const int tl = row >> 4, rr = row & 15;
                const int64_t si = ((int64_t(it.e) * nrb + it.rb) * kTilesPerBlock + tl) * 16 + (rr & 7) * 2 + (rr >> 3);
                s = a.scale_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(a.S)[si])
                                 : reinterpret_cast<const float*>(a.S)[si];
            }
            const float bias = (a.bias && valid) ? a.bias[int64_t(it.e) * a.N + prow] : 0.0f;
            const uint32_t tbase = tmem + (uint32_t(qd * 32) << 16) + uint32_t(acc * BNMAX);
            const int ncol = ((it.rows + 15) / 16) * 16;
            const bool empty_k = it.ks_hi <= it.ks_lo;  // no MMA wrote the accumulator
            for (int c0 = 16 * half; c0 < ncol; c0 += 32) {
                float v[16];
                tmem_ld16(tbase + uint32_t(c0), v);
                if (empty_k)
#pragma unroll
                    for (int j = 0; j < 16; ++j) v[j] = 0.0f;
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int col = c0 + j;
                    const float val = fmaf(v[j], s, bias);
                    const bool in = col < it.rows;
                    const int64_t p = it.seg0 + int64_t(it.tt) * a.bn + col;  // permuted row
                    if (a.is_fc1) {
                        if (a.gated) {
                            const float up = __shfl_down_sync(0xffffffffu, val, 8);
                            if (in && valid && (row & 15) < 8) {
                                const int64_t I = a.N / 2;
                                const int64_t ii = (prow >> 4) * 8 + (row & 7);
                                reinterpret_cast<__nv_bfloat16*>(a.out)[p * I + ii] =
                                    __float2bfloat16_rn(act_gated(a.act_type, val, up, a.alpha, a.beta, a.limit));
                            }
                        } else if (in && valid) {
                            reinterpret_cast<__nv_bfloat16*>(a.out)[p * a.N + prow] =
                                __float2bfloat16_rn(act_plain(a.act_type, val));
                        }
                    } else if (in && valid) {
                        reinterpret_cast<float*>(a.out)[(int64_t(it.split) * a.R + p) * a.N + prow] = val;
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&acce[acc]));
            if (++acc == 2) { acc = 0; aph ^= 1u; }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::kTmemCols));
    }
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

template <int BITS, bool PERCOL, int BNMAX>
struct Launch {
    static constexpr int kStage = TcCfg<BITS, PERCOL, BNMAX, 1>::kStage;
    static constexpr int kByTmem = (512 - 2 * BNMAX) / kAStageCols;
    static constexpr int kBySmem = (200 * 1024) / kStage;
    static constexpr int kStages = kByTmem < kBySmem ? (kByTmem < 12 ? kByTmem : 12) : (kBySmem < 12 ? kBySmem : 12);
    using C = TcCfg<BITS, PERCOL, BNMAX, kStages>;
    static cudaError_t prepare() {
        return cudaFuncSetAttribute(ffn_tc_kernel<BITS, PERCOL, BNMAX, kStages>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    }
    static cudaError_t run(const CUtensorMap& map, const TcArgs& a, int grid, cudaStream_t st) {
        ffn_tc_kernel<BITS, PERCOL, BNMAX, kStages><<<grid, kTcThreads, C::kSmem, st>>>(map, a);
        return cudaGetLastError();
    }
};

template <int BITS, bool PERCOL>
cudaError_t dispatch_bn(int bnmax, const CUtensorMap& map, const TcArgs& a, int grid, cudaStream_t st) {
    switch (bnmax) {
        case 16: return Launch<BITS, PERCOL, 16>::run(map, a, grid, st);
        case 32: return Launch<BITS, PERCOL, 32>::run(map, a, grid, st);
        case 64: return Launch<BITS, PERCOL, 64>::run(map, a, grid, st);
        default: return Launch<BITS, PERCOL, 128>::run(map, a, grid, st);
    }
}

template <int BITS, bool PERCOL>
cudaError_t prepare_bits() {
    cudaError_t e = Launch<BITS, PERCOL, 16>::prepare();
    if (e == cudaSuccess) e = Launch<BITS, PERCOL, 32>::prepare();
    if (e == cudaSuccess) e = Launch<BITS, PERCOL, 64>::prepare();
    if (e == cudaSuccess) e = Launch<BITS, PERCOL, 128>::prepare();
    return e;
}

__global__ void gather_rows_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ perm,
                                   uint4* __restrict__ xp, int64_t R, int64_t row_vecs) {
    const int64_t total = R * row_vecs;
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < total;
         i += int64_t(gridDim.x) * blockDim.x) {
        const int64_t p = i / row_vecs, v = i - p * row_vecs;
        xp[i] = x[int64_t(perm[p]) * row_vecs + v];
    }
}


// ==========================================================================
// Streaming decode on the tensor cores (few routed rows per expert).
//
// Same dequantise-into-TMEM scheme, organised for weight streaming:
//   * work items (expert, token tile, K-split, 128-row block) are handed to
//     CTAs in contiguous runs, so consecutive items share their activations;
//     those ([tile rows x K-split range] bf16) are loaded once per run with a
//     single 3-D TMA into shared memory and stay resident;
//   * a stage is 128 k: one bulk copy of 8 KB (int4) / 16 KB (int8) of
//     packed codes, in a ring of its own that the dequantise warps release as
//     soon as they have read it, so HBM streaming never waits on the MMAs;
//   * decoded A tiles go to a separate ring of TMEM slots (64 columns each)
//     that the MMA completions release;
//   * a stage's block scales ride in the same ring slot (a second bulk copy
//     on the same barrier), so no dequantise warp waits on a global load.
// ==========================================================================
constexpr int kDBK = 128;                 // k per streaming stage
constexpr int kDAStageCols = kDBK / 2;    // TMEM columns of one A tile
// warps: 16 dequantise (two per 16-row tile, taking alternate stages),
// producer, MMA, 4 epilogue
constexpr int kDDeqWarps = 16;
constexpr int kDWarpProd = 16;
constexpr int kDWarpMma = 17;
constexpr int kDThreads = 22 * 32;
constexpr int kDEpiWarps = 4;

constexpr int kDRingMax = 8;              // packed-ring slots at most
constexpr int kDBMax = 128 * 1024;        // resident activations
constexpr int kDBarBytes = 3072;          // barriers, TMEM slot, item prefix
constexpr int kDSmemMax = 227 * 1024;

template <int BITS, bool PERCOL, int BN>
struct TcdCfg {
    static constexpr int kPacked = kBlockRows * kDBK * BITS / 8;  // 8 KB / 16 KB
    static constexpr int kAStages = (512 - 2 * BN) / kDAStageCols; // 7 / 6
    static constexpr int kACol0 = 2 * BN;
};

// Bytes of one stage's block scales (128 rows x the scale blocks of 128 k).
__host__ __device__ inline int tcd_scale_bytes(int block_size, int scale_bf16) {
    if (block_size == 0) return 0;
    const int nsb = block_size >= kDBK ? 1 : kDBK / block_size;
    return nsb * kBlockRows * (scale_bf16 ? 2 : 4);
}

// Item order: expert, token tile, split, row block (row block fastest).
__device__ __forceinline__ Item item_at_stream(int i, const int* prefix, const TcArgs& a, int nrb, int nks) {
    int lo = 0, hi = a.E;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (prefix[mid] <= i) lo = mid; else hi = mid;
    }
    Item it;
    it.e = lo;
    it.seg0 = a.offsets[lo];
    it.M = a.offsets[lo + 1] - int(it.seg0);
    int rem = i - prefix[lo];
    const int per_tt = a.splits * nrb;
    it.tt = rem / per_tt;
    rem -= it.tt * per_tt;
    it.split = rem / nrb;
    it.rb = rem - it.split * nrb;
    it.rows = min(a.bn, it.M - it.tt * a.bn);
    it.ks_lo = int((int64_t(it.split) * nks) / a.splits);
    it.ks_hi = int((int64_t(it.split + 1) * nks) / a.splits);
    return it;
}

__device__ __forceinline__ void tma_3d(uint32_t dst, const CUtensorMap* map, int x, int y, int z,
                                       uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, "
        "{%2, %3, %4}], [%5];" ::"r"(dst),
        "l"(map), "r"(x), "r"(y), "r"(z), "r"(bar)
        : "memory");
}


template <int BITS, bool PERCOL, int BN>
__global__ void __launch_bounds__(kDThreads, 1)
    ffn_tc_decode_kernel(const __grid_constant__ CUtensorMap bmap, const TcArgs a) {
    using C = TcdCfg<BITS, PERCOL, BN>;
    constexpr int AS = C::kAStages;
    const int PS = a.ring, SLOT = a.stage_bytes;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint8_t* bsm = smem;                           // resident activations [chunk][BN rows][128 B]
    uint8_t* psm = smem + kDBMax + kDBarBytes;     // ring: [packed codes][block scales] per slot
    uint64_t* pfull = reinterpret_cast<uint64_t*>(smem + kDBMax);
    uint64_t* pempty = pfull + kDRingMax;
    uint64_t* afull = pempty + kDRingMax;
    uint64_t* aempty = afull + AS;
    uint64_t* accf = aempty + AS;
    uint64_t* acce = accf + 2;
    uint64_t* bfull = acce + 2;
    uint64_t* bempty = bfull + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bempty + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* prefix = reinterpret_cast<int*>(tmem_slot + 4);

    const int nrb = int(padded_rows(a.N) / kBlockRows);
    const int nks = int(a.K / kDBK);

    if (tid == 0) {
        for (int s = 0; s < PS; ++s) {
            mbar_init(smem_u32(&pfull[s]), 1);
            mbar_init(smem_u32(&pempty[s]), kDeqWarps);
        }
        for (int s = 0; s < AS; ++s) {
            mbar_init(smem_u32(&afull[s]), kDeqWarps);
            mbar_init(smem_u32(&aempty[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&accf[b]), 1);
            mbar_init(smem_u32(&acce[b]), kDEpiWarps);
        }
        mbar_init(smem_u32(bfull), 1);
        mbar_init(smem_u32(bempty), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        int carry = 0;
        for (int e0 = 0; e0 < a.E; e0 += 32) {
            const int e = e0 + lane;
            int v = 0;
            if (e < a.E) {
                const int M = a.offsets[e + 1] - a.offsets[e];
                v = ((M + a.bn - 1) / a.bn) * nrb * a.splits;
            }
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += n;
            }
            if (e < a.E) prefix[e] = carry + incl - v;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) prefix[a.E] = carry;
    }
    if (warp == kDWarpMma) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(512));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int total = prefix[a.E];
    // contiguous run of items for this CTA
    const int i_lo = int((int64_t(blockIdx.x) * total) / gridDim.x);
    const int i_hi = int((int64_t(blockIdx.x + 1) * total) / gridDim.x);
    auto same_b = [](const Item& p, const Item& q) {
        return p.e == q.e && p.tt == q.tt && p.split == q.split;
    };

    if (warp == kDWarpProd) {
        {
            const uint32_t e = elect_one();
            int ps = 0;
            uint32_t pph = 0, bph = 0;
            bool ok = true;
            const int ngr = int(a.K / kgroup_of(BITS));
            const int sbytes = PERCOL ? 0 : tcd_scale_bytes(a.block_size, a.scale_bf16);
            const int nsb = PERCOL ? 1 : int(a.K / a.block_size);
            const int ssz = a.scale_bf16 ? 2 : 4;
            Item prev{};
            prev.e = -1;
            for (int i = i_lo; ok && i < i_hi; ++i) {
                const Item it = item_at_stream(i, prefix, a, nrb, nks);
                if (prev.e < 0 || !same_b(prev, it)) {
                    // activations of this run: [rows, ks_lo*128 .. ks_hi*128) as 64-k chunks
                    if (!warp_wait(smem_u32(bempty), bph ^ 1u, abort_flag, a.status)) { ok = false; break; }
                    bph ^= 1u;
                    // the box always spans the largest split (OOB rows/chunks arrive as zeros)
                    const int box_ch = ((nks + a.splits - 1) / a.splits) * (kDBK / 64);
                    mbar_expect_tx_e(smem_u32(bfull), uint32_t(box_ch * BN * 128), e);
                    tma_3d_e(smem_u32(bsm), &bmap, 0, int(it.seg0) + it.tt * a.bn, it.ks_lo * (kDBK / 64),
                             smem_u32(bfull), e);
                }
                prev = it;
                for (int ks = it.ks_lo; ks < it.ks_hi; ++ks) {
                    if (!warp_wait(smem_u32(&pempty[ps]), pph ^ 1u, abort_flag, a.status)) { ok = false; break; }
                    const uint32_t fb = smem_u32(&pfull[ps]);
                    mbar_expect_tx_e(fb, uint32_t(C::kPacked + sbytes), e);
                    const int g = ks * (kDBK / kgroup_of(BITS));
                    const uint8_t* src =
                        a.W + ((int64_t(it.e) * nrb + it.rb) * ngr + g) * int64_t(kTilesPerBlock) * kUnitBytes;
                    uint8_t* slot = psm + ps * SLOT;
                    bulk_g2s_e(smem_u32(slot), src, C::kPacked, fb, e);
                    if (!PERCOL) {
                        // scale blocks [sb0, sb0 + n) of this row block: contiguous, 128 per block
                        const int64_t sb0 = (int64_t(ks) * kDBK) / a.block_size;
                        const int64_t off = ((int64_t(it.e) * nrb + it.rb) * nsb + sb0) * kBlockRows * ssz;
                        bulk_g2s_e(smem_u32(slot + C::kPacked), static_cast<const uint8_t*>(a.S) + off,
                                   uint32_t(sbytes), fb, e);
                    }
                    if (++ps == PS) { ps = 0; pph ^= 1u; }
                }
            }
        }
    } else if (warp == kDWarpMma) {
        {
            const uint32_t e = elect_one();
            int as = 0, acc = 0;
            uint32_t aph = 0, cph = 0, bph = 0;
            bool ok = true;
            Item prev{};
            prev.e = -1;
            const uint32_t b0 = smem_u32(bsm);
            for (int i = i_lo; ok && i < i_hi; ++i) {
                const Item it = item_at_stream(i, prefix, a, nrb, nks);
                if (prev.e < 0 || !same_b(prev, it)) {
                    if (!warp_wait(smem_u32(bfull), bph, abort_flag, a.status)) break;
                    bph ^= 1u;
                }
                prev = it;
                const int n = ((it.rows + 15) / 16) * 16;
                const uint32_t idesc = idesc_bf16(n);
                if (!warp_wait(smem_u32(&acce[acc]), cph ^ 1u, abort_flag, a.status)) break;
                tc_fence_after();
                const uint32_t d = tmem + uint32_t(acc * BN);
                for (int ks = it.ks_lo; ks < it.ks_hi; ++ks) {
                    if (!warp_wait(smem_u32(&afull[as]), aph, abort_flag, a.status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t at = tmem + uint32_t(C::kACol0 + as * kDAStageCols);
                    // first 64-k chunk of this stage in the resident activations
                    const uint64_t bd = desc_sw128(b0 + uint32_t((ks - it.ks_lo) * (kDBK / 64) * BN * 128));
                    const uint32_t acc0 = ks > it.ks_lo ? 1u : 0u;
#pragma unroll
                    for (int kk = 0; kk < kDBK / 16; ++kk) {
                        // chunk kk/4 (BN rows of 128 B each), 32 B per 16 k inside the swizzled row
                        const uint64_t bk = bd + uint64_t(((kk / 4) * BN * 128 + 32 * (kk % 4)) >> 4);
                        mma_bf16_ts_e(d, at + uint32_t(8 * kk), bk, idesc, kk > 0 ? 1u : acc0, e);
                    }
                    mma_commit_e(smem_u32(&aempty[as]), e);
                    if (++as == AS) { as = 0; aph ^= 1u; }
                }
                if (!ok) break;
                mma_commit_e(smem_u32(&accf[acc]), e);
                if (++acc == 2) { acc = 0; cph ^= 1u; }
                // release the resident activations after the run's last item
                bool last = i + 1 >= i_hi;
                if (!last) last = !same_b(it, item_at_stream(i + 1, prefix, a, nrb, nks));
                if (last) mma_commit_e(smem_u32(bempty), e);
            }
        }
    } else if (warp < kDDeqWarps) {
        // tile: TMEM lanes 16*tile.. lie in this warp's lane quarter (warp % 4);
        // par: this warp takes the stages of that parity (stage count in the CTA)
        const int tile = 2 * (warp & 3) + ((warp >> 2) & 1);
        const int par = warp >> 3;
        const int r0 = lane >> 2, c = lane & 3;
        const uint32_t lane_addr = uint32_t(16 * tile) << 16;
        int ps = par, as = par;  // both rings have at least two slots
        uint32_t pph = 0, aph = 0;
        int sn = 0;
        bool ok = true;
        const uint32_t kMask = 0x000F000Fu, kMagic = 0x43004300u, kBias4 = 0x43084308u;
        constexpr int GROUPS = kDBK / kgroup_of(BITS);  // 2 (int4) or 4 (int8)
        constexpr int KSTEPS = kgroup_of(BITS) / 16;
        // this lane's pair of rows (r0, r0 + 8) inside one scale block of the slot
        const int srow = tile * 16 + 2 * r0;
        // scale block (relative to the stage) of a k offset; with blocks of
        // 128 k or more, one block covers the whole stage
        const int bs_shift = a.block_size >= kDBK ? 30 : __ffs(a.block_size) - 1;
        for (int i = i_lo; ok && i < i_hi; ++i) {
            const Item it = item_at_stream(i, prefix, a, nrb, nks);
            for (int ks = it.ks_lo; ks < it.ks_hi; ++ks) {
                if (((sn++) & 1) != par) continue;
                if (!warp_wait(smem_u32(&pfull[ps]), pph, abort_flag, a.status)) { ok = false; break; }
                uint4 wq[GROUPS];
                const uint8_t* pk = psm + ps * SLOT;
#pragma unroll
                for (int gg = 0; gg < GROUPS; ++gg)
                    wq[gg] = *reinterpret_cast<const uint4*>(pk + ((gg * kTilesPerBlock + tile) * 32 + lane) * 16);
                float sA[GROUPS][KSTEPS], sB[GROUPS][KSTEPS];
                if (!PERCOL) {
                    const uint8_t* sk = pk + C::kPacked;
#pragma unroll
                    for (int gg = 0; gg < GROUPS; ++gg)
#pragma unroll
                        for (int j = 0; j < KSTEPS; ++j) {
                            const int kl = gg * kgroup_of(BITS) + 16 * j + 4 * c;
                            const int si = ((kl >> bs_shift) << 7) + srow;
                            if (a.scale_bf16) {
                                const uint32_t raw = *reinterpret_cast<const uint32_t*>(sk + 2 * si);
                                sA[gg][j] = __uint_as_float(raw << 16);
                                sB[gg][j] = __uint_as_float(raw & 0xFFFF0000u);
                            } else {
                                const float2 f = *reinterpret_cast<const float2*>(sk + 4 * si);
                                sA[gg][j] = f.x;
                                sB[gg][j] = f.y;
                            }
                        }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&pempty[ps]));
                ps += 2;
                if (ps >= PS) { ps -= PS; pph ^= 1u; }
                if (!warp_wait(smem_u32(&aempty[as]), aph ^ 1u, abort_flag, a.status)) { ok = false; break; }
                tc_fence_after();
                const uint32_t at = tmem + lane_addr + uint32_t(C::kACol0 + as * kDAStageCols);
#pragma unroll
                for (int gg = 0; gg < GROUPS; ++gg) {
                    const uint32_t wv[4] = {wq[gg].x, wq[gg].y, wq[gg].z, wq[gg].w};
                    uint32_t r[4 * KSTEPS];
#pragma unroll
                    for (int j = 0; j < KSTEPS; ++j) {
                        uint32_t A[4];
                        if (BITS == 4) {
                            A[0] = bf2_sub((wv[j] & kMask) | kMagic, kBias4);
                            A[1] = bf2_sub(((wv[j] >> 4) & kMask) | kMagic, kBias4);
                            A[2] = bf2_sub(((wv[j] >> 8) & kMask) | kMagic, kBias4);
                            A[3] = bf2_sub(((wv[j] >> 12) & kMask) | kMagic, kBias4);
                        } else {
#pragma unroll
                            for (int qq = 0; qq < 4; ++qq) {
                                const uint32_t word = wv[2 * j + (qq >> 1)];
                                const uint32_t pr = __byte_perm(word, 0u, (qq & 1) ? 0x4342u : 0x4140u);
                                const uint32_t lo = (pr & 0x007F007Fu) | 0x43004300u;
                                const uint32_t hi = (pr & 0x00800080u) ^ 0x43804380u;
                                A[qq] = bf2_sub(lo, hi);
                            }
                        }
                        if (!PERCOL) {
                            const uint32_t sa2 = bf2_bcast(sA[gg][j]), sb2 = bf2_bcast(sB[gg][j]);
                            A[0] = bf2_mul(A[0], sa2);
                            A[2] = bf2_mul(A[2], sa2);
                            A[1] = bf2_mul(A[1], sb2);
                            A[3] = bf2_mul(A[3], sb2);
                        }
                        r[4 * j + 0] = A[0];
                        r[4 * j + 1] = A[2];
                        r[4 * j + 2] = A[1];
                        r[4 * j + 3] = A[3];
                    }
                    // k-group gg of the stage covers TMEM columns [gg*KG/2, (gg+1)*KG/2)
                    if (BITS == 4)
                        tmem_st16x256_x4(at + uint32_t(gg * 32), *reinterpret_cast<const uint32_t(*)[16]>(r));
                    else
                        tmem_st16x256_x2(at + uint32_t(gg * 16), *reinterpret_cast<const uint32_t(*)[8]>(r));
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&afull[as]));
                as += 2;
                if (as >= AS) { as -= AS; aph ^= 1u; }
            }
        }
    } else {
        // epilogue: warps 18..21, one per TMEM lane quarter
        const int qd = warp & 3;
        const int row = qd * 32 + lane;
        int acc = 0;
        uint32_t cph = 0;
        for (int i = i_lo; i < i_hi; ++i) {
            const Item it = item_at_stream(i, prefix, a, nrb, nks);
            if (!warp_wait(smem_u32(&accf[acc]), cph, abort_flag, a.status)) break;
            tc_fence_after();
            const int64_t prow = int64_t(it.rb) * kBlockRows + row;
            const bool valid = prow < a.N;
            float s = 1.0f;
            if (PERCOL && valid) {
                const int tl = row >> 4, rr = row & 15;
                const int64_t si = ((int64_t(it.e) * nrb + it.rb) * kTilesPerBlock + tl) * 16 + (rr & 7) * 2 + (rr >> 3);
                s = a.scale_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(a.S)[si])
                                 : reinterpret_cast<const float*>(a.S)[si];
            }
            const float bias = (a.bias && valid) ? a.bias[int64_t(it.e) * a.N + prow] : 0.0f;
            const uint32_t tbase = tmem + (uint32_t(qd * 32) << 16) + uint32_t(acc * BN);
            const int ncol = ((it.rows + 15) / 16) * 16;
            const bool empty_k = it.ks_hi <= it.ks_lo;  // no MMA wrote the accumulator
            for (int c0 = 0; c0 < ncol; c0 += 16) {
                float v[16];
                tmem_ld16(tbase + uint32_t(c0), v);
                if (empty_k)
#pragma unroll
                    for (int j = 0; j < 16; ++j) v[j] = 0.0f;
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int col = c0 + j;
                    const float val = fmaf(v[j], s, bias);
                    const bool in = col < it.rows;
                    const int64_t p = it.seg0 + int64_t(it.tt) * a.bn + col;
                    if (a.is_fc1) {
                        if (a.gated) {
                            const float up = __shfl_down_sync(0xffffffffu, val, 8);
                            if (in && valid && (row & 15) < 8) {
                                const int64_t I = a.N / 2;
                                const int64_t ii = (prow >> 4) * 8 + (row & 7);
                                reinterpret_cast<__nv_bfloat16*>(a.out)[p * I + ii] =
                                    __float2bfloat16_rn(act_gated(a.act_type, val, up, a.alpha, a.beta, a.limit));
                            }
                        } else if (in && valid) {
                            reinterpret_cast<__nv_bfloat16*>(a.out)[p * a.N + prow] =
                                __float2bfloat16_rn(act_plain(a.act_type, val));
                        }
                    } else if (in && valid) {
                        reinterpret_cast<float*>(a.out)[(int64_t(it.split) * a.R + p) * a.N + prow] = val;
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&acce[acc]));
            if (++acc == 2) { acc = 0; cph ^= 1u; }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kDWarpMma) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
    }
}

template <int BITS, bool PERCOL, int BN>
struct LaunchD {
    static cudaError_t prepare() {
        return cudaFuncSetAttribute(ffn_tc_decode_kernel<BITS, PERCOL, BN>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, kDSmemMax);
    }
    static cudaError_t run(const CUtensorMap& map, const TcArgs& a, int grid, cudaStream_t st) {
        const int smem = 1024 + kDBMax + kDBarBytes + a.ring * a.stage_bytes;
        ffn_tc_decode_kernel<BITS, PERCOL, BN><<<grid, kDThreads, smem, st>>>(map, a);
        return cudaGetLastError();
    }
};

template <int BITS, bool PERCOL>
cudaError_t prepare_bits_d() {
    cudaError_t e = LaunchD<BITS, PERCOL, 16>::prepare();
    if (e == cudaSuccess) e = LaunchD<BITS, PERCOL, 32>::prepare();
    return e;
}

}  // namespace

cudaError_t prepare_ffn_tc() {
    cudaError_t e = prepare_bits<4, false>();
    if (e == cudaSuccess) e = prepare_bits<4, true>();
    if (e == cudaSuccess) e = prepare_bits<8, false>();
    if (e == cudaSuccess) e = prepare_bits<8, true>();
    if (e == cudaSuccess) e = prepare_bits_d<4, false>();
    if (e == cudaSuccess) e = prepare_bits_d<4, true>();
    if (e == cudaSuccess) e = prepare_bits_d<8, false>();
    if (e == cudaSuccess) e = prepare_bits_d<8, true>();
    return e;
}

bool tc_decode_fits(int64_t K, int splits, int bn) {
    if (K % kDBK != 0 || bn > 32) return false;
    const int64_t nks = K / kDBK;
    const int64_t per = (nks + splits - 1) / splits;  // largest split, in stages
    const int bnr = bn <= 16 ? 16 : 32;
    return per * kDBK * 2 * bnr <= 128 * 1024;
}

cudaError_t launch_ffn_tc_decode(const FfnArgs& f, int bn, int32_t* status, cudaStream_t st) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    const int bnr = bn <= 16 ? 16 : 32;
    if (!tc_decode_fits(f.K, f.splits, bn)) return cudaErrorInvalidValue;
    // activations viewed as [K/64 chunks][rows][64]: box = (64, bnr rows, chunks of a split)
    const int64_t nks = f.K / kDBK;
    const int64_t per = (nks + f.splits - 1) / f.splits;
    CUtensorMap map;
    const cuuint64_t dims[3] = {cuuint64_t(64), cuuint64_t(f.R), cuuint64_t(f.K / 64)};
    const cuuint64_t strides[2] = {cuuint64_t(f.K * 2), cuuint64_t(128)};
    const cuuint32_t box[3] = {cuuint32_t(64), cuuint32_t(bnr), cuuint32_t(per * (kDBK / 64))};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(f.act), dims, strides, box,
                     estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    TcArgs a{};
    a.W = f.W;
    a.S = f.S;
    a.bias = f.bias;
    a.offsets = f.offsets;
    a.out = f.out;
    a.status = status;
    a.N = f.N;
    a.K = f.K;
    a.R = f.R;
    a.E = f.E;
    a.block_size = f.block_size;
    a.gated = f.gated;
    a.is_fc1 = f.is_fc1;
    a.act_type = f.act_type;
    a.alpha = f.alpha;
    a.beta = f.beta;
    a.limit = f.limit;
    a.splits = f.splits;
    a.scale_bf16 = f.scale_bf16;
    a.bn = bn;
    {
        // ring slot: packed codes then block scales, rounded to 128 B; as many
        // slots (up to 8) as the shared memory left beside the activations holds
        const int packed = kBlockRows * kDBK * f.bits / 8;
        a.stage_bytes = (packed + tcd_scale_bytes(f.block_size, f.scale_bf16) + 127) & ~127;
        const int room = kDSmemMax - 1024 - kDBMax - kDBarBytes;
        a.ring = std::min(f.bits == 4 ? kDRingMax : 4, room / a.stage_bytes);
        if (a.ring < 2) return cudaErrorInvalidValue;
    }
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const bool percol = f.block_size == 0;
    if (f.bits == 4) {
        if (bnr == 16) return percol ? LaunchD<4, true, 16>::run(map, a, sms, st) : LaunchD<4, false, 16>::run(map, a, sms, st);
        return percol ? LaunchD<4, true, 32>::run(map, a, sms, st) : LaunchD<4, false, 32>::run(map, a, sms, st);
    }
    if (bnr == 16) return percol ? LaunchD<8, true, 16>::run(map, a, sms, st) : LaunchD<8, false, 16>::run(map, a, sms, st);
    return percol ? LaunchD<8, true, 32>::run(map, a, sms, st) : LaunchD<8, false, 32>::run(map, a, sms, st);
}

cudaError_t launch_gather_rows(const void* x, const int32_t* perm, void* xp, int64_t R, int64_t row_bytes,
                               cudaStream_t st) {
    if (R == 0) return cudaSuccess;
    const int64_t vecs = row_bytes / 16;
    int64_t blocks = (R * vecs + 255) / 256;
    if (blocks > 148 * 8) blocks = 148 * 8;
    gather_rows_kernel<<<unsigned(blocks), 256, 0, st>>>(reinterpret_cast<const uint4*>(x), perm,
                                                       reinterpret_cast<uint4*>(xp), R, vecs);
    return cudaGetLastError();
}

cudaError_t launch_ffn_tc(const FfnArgs& f, int bn, int32_t* status, cudaStream_t st) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    int bnmax = 16;
    while (bnmax < bn) bnmax *= 2;
    if (bnmax > 128) return cudaErrorInvalidValue;
    // activations: [rows, K] bf16; rows = R (permuted rows)
    const int64_t rows = f.R;
    CUtensorMap map;
    const cuuint64_t dims[2] = {cuuint64_t(f.K), cuuint64_t(rows)};
    const cuuint64_t strides[1] = {cuuint64_t(f.K * 2)};
    const cuuint32_t box[2] = {cuuint32_t(kBK), cuuint32_t(bnmax < 64 ? bnmax : 64)};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(f.act), dims, strides, box,
                     estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    TcArgs a{};
    a.W = f.W;
    a.S = f.S;
    a.bias = f.bias;
    a.offsets = f.offsets;
    a.out = f.out;
    a.status = status;
    a.N = f.N;
    a.K = f.K;
    a.R = f.R;
    a.E = f.E;
    a.block_size = f.block_size;
    a.gated = f.gated;
    a.is_fc1 = f.is_fc1;
    a.act_type = f.act_type;
    a.alpha = f.alpha;
    a.beta = f.beta;
    a.limit = f.limit;
    a.splits = f.splits;
    a.scale_bf16 = f.scale_bf16;
    a.bn = bn;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const bool percol = f.block_size == 0;
    if (f.bits == 4)
        return percol ? dispatch_bn<4, true>(bnmax, map, a, sms, st) : dispatch_bn<4, false>(bnmax, map, a, sms, st);
    return percol ? dispatch_bn<8, true>(bnmax, map, a, sms, st) : dispatch_bn<8, false>(bnmax, map, a, sms, st);
}

}  // namespace qmoe
