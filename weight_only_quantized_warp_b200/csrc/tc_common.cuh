// tc_common.cuh -- pieces shared by the tcgen05 expert-FFN kernels (sm_100a):
// kernel arguments, mbarrier / bulk-copy / TMA / tcgen05 PTX wrappers, bf16x2
// arithmetic, activations, work-item record and the tensor-map encoder entry
// point. Everything is internal to the including translation unit.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "qmoe_internal.cuh"

namespace qmoe {
namespace {

// Default limit of every bounded device wait (QMOE_OPT_WAIT_LIMIT_NS).
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
    int ring, stage_bytes, sring;  // streaming decode: packed-ring slots, scale-slot bytes, scale-ring slots
    uint64_t timeout_ns;     // limit of every bounded wait
    int withhold;            // test only: the MMA warp keeps back its first item's accumulator signal
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

// Potentially blocking test: a warp whose phase is still open is suspended
// (it issues nothing) until the phase completes or kSuspendNs pass.
constexpr uint32_t kSuspendNs = 10000;

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
        "selp.b32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(kSuspendNs)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t now_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Non-blocking test of a phase (no suspension when the phase is still open).
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n.reg .pred p;\nmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        "selp.b32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait on a phase parity. Returns false (after raising the CTA's
// abort flag and the workspace status) when the wait gives up after
// limit_ns, or another role already aborted.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          int32_t* status, uint64_t limit_ns) {
    if (mbar_test(bar, parity)) return true;
    const uint64_t t0 = now_ns();
    for (uint32_t spin = 1;; ++spin) {
        if (mbar_try(bar, parity)) return true;
        if ((spin & 15u) == 0u) {
            if (*abort_flag) return false;
            if (now_ns() - t0 > limit_ns) {
                *abort_flag = 1;
                atomicExch(status, int32_t(QMOE_TIMEOUT));
                return false;
            }
        }
    }
}

// Run of completed phases, by a whole warp without blocking: tests the ring
// stages st, st + step, ... (up to L of them, the parity flipping where the
// ring wraps) on bars0 (and bars1 when given) and returns how many leading
// ones have completed. The tests are independent, so their shared-memory
// round trips overlap; a role that finds several stages ready consumes them
// without testing again. Valid while the stages tested lie within one lap of
// the ring: (L - 1) * step < stages. Lane 0's view is taken by every lane.
template <int L>
__device__ __forceinline__ int ready_run(const uint64_t* bars0, const uint64_t* bars1, int st, uint32_t parity,
                                         int step, int stages) {
    uint32_t mask = 0;
#pragma unroll
    for (int j = 0; j < L; ++j) {
        bool ok = mbar_test(smem_u32(&bars0[st]), parity);
        if (bars1 != nullptr) ok = mbar_test(smem_u32(&bars1[st]), parity) & ok;
        mask |= uint32_t(ok) << j;
        st += step;
        if (st >= stages) {
            st -= stages;
            parity ^= 1u;
        }
    }
    mask = __shfl_sync(0xffffffffu, mask, 0);
    return __ffs(~mask) - 1;
}

// Wait by a whole warp: every lane polls, and the warp continues only if all
// lanes saw the phase complete (a timeout in any lane stops the whole warp).
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          int32_t* status, uint64_t limit_ns) {
    const bool ok = mbar_wait(bar, parity, abort_flag, status, limit_ns);
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

__device__ __forceinline__ void mma_bf16_ss_e(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                              uint32_t accumulate, uint32_t e) {
    asm volatile(
        "{\n.reg .pred p, q;\nsetp.ne.b32 p, %4, 0;\nsetp.ne.b32 q, %5, 0;\n"
        "@q tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(e));
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
        case kActGeluTanh: return 0.5f * a * (1.0f + tanhf(0.79788456080286536f * (a + 0.044715f * a * a * a)));
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

// Epilogue of one work item for the thread that owns accumulator lane `row`
// (packed row rb*128 + row of the item's expert): columns c_first,
// c_first + c_step, ... in chunks of 16 from the accumulator at TMEM address
// tbase; scale (per-column mode), bias, activation and the store of h (FC1)
// or of the split's fp32 partial (FC2).
template <bool PERCOL>
__device__ __forceinline__ void tc_epilogue_item(const TcArgs& a, const Item& it, int nrb, uint32_t tbase, int row,
                                                 int lane, int c_first, int c_step) {
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
    const int ncol = ((it.rows + 15) / 16) * 16;
    const bool empty_k = it.ks_hi <= it.ks_lo;  // no MMA wrote the accumulator
    const int64_t p0 = it.seg0 + int64_t(it.tt) * a.bn;  // permuted row of column 0
    if (a.is_fc1 && a.gated) {
        // tile rows 0-7 are gate rows, 8-15 the matching up rows (lane ^ 8):
        // each lane of a pair finishes half of every 16 columns, so all
        // lanes compute activations
        const bool gate_lane = (lane & 8) == 0;
        const int64_t I = a.N / 2;
        __nv_bfloat16* hout = reinterpret_cast<__nv_bfloat16*>(a.out) + p0 * I + (prow >> 4) * 8 + (row & 7);
        // decided once per item (uniform over the warp): the scale/bias pass
        // only where a scale or a bias exists, SwiGLU inline, its clamps only
        // for a finite limit
        const bool affine = PERCOL || a.bias != nullptr;
        const bool swiglu = a.act_type == QMOE_ACT_SWIGLU;
        const bool clamp = swiglu && a.limit < INFINITY;
        const int ncols = valid ? it.rows : 0;  // columns this lane stores
        const int coff = gate_lane ? 0 : 8;
        for (int c0 = c_first; c0 < ncol; c0 += c_step) {
            float v[16];
            tmem_ld16(tbase + uint32_t(c0), v);
            if (empty_k) {
#pragma unroll
                for (int j = 0; j < 16; ++j) v[j] = 0.0f;
            } else if (affine) {
#pragma unroll
                for (int j = 0; j < 16; ++j) v[j] = fmaf(v[j], s, bias);
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float recv = __shfl_xor_sync(0xffffffffu, gate_lane ? v[j + 8] : v[j], 8);
                float g = gate_lane ? v[j] : recv;
                float u = gate_lane ? recv : v[j + 8];
                const int col = c0 + j + coff;
                float hv;
                if (swiglu) {
                    if (clamp) {
                        g = fminf(g, a.limit);
                        u = fminf(fmaxf(u, -a.limit), a.limit);
                    }
                    hv = (u + a.beta) * g * sigmoidf_(a.alpha * g);
                } else {
                    hv = act_gated(a.act_type, g, u, a.alpha, a.beta, a.limit);
                }
                if (col < ncols) hout[int64_t(col) * I] = __float2bfloat16_rn(hv);
            }
        }
    } else {
        const bool affine = PERCOL || a.bias != nullptr;
        const int ncols = valid ? it.rows : 0;  // columns this lane stores
        for (int c0 = c_first; c0 < ncol; c0 += c_step) {
            float v[16];
            tmem_ld16(tbase + uint32_t(c0), v);
            if (empty_k) {
#pragma unroll
                for (int j = 0; j < 16; ++j) v[j] = 0.0f;
            } else if (affine) {
#pragma unroll
                for (int j = 0; j < 16; ++j) v[j] = fmaf(v[j], s, bias);
            }
            if (a.is_fc1) {
                __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(a.out) + (p0 + c0) * a.N + prow;
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    if (c0 + j < ncols) o[int64_t(j) * a.N] = __float2bfloat16_rn(act_plain(a.act_type, v[j]));
            } else {
                // FC2: this split's fp32 partial of permuted rows p0 + c0 + j
                float* o = reinterpret_cast<float*>(a.out) + (int64_t(it.split) * a.R + p0 + c0) * a.N + prow;
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    if (c0 + j < ncols) o[int64_t(j) * a.N] = v[j];
            }
        }
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

}  // namespace
}  // namespace qmoe
