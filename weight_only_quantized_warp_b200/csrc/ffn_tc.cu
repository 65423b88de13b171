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
// Warp roles of one persistent CTA (864 threads, one CTA per SM):
//   warps 0-15  dequantise: packed codes (shared) -> bf16 A tile written
//               straight into tensor memory (tcgen05.st), one 16-row tile per
//               warp; two groups of eight warps take alternate stages, so two
//               stages are decoded at once; the A operand never touches
//               shared memory
//   warp 16     activation producer: 64-row TMA boxes of the activations
//               (bf16, 128-byte swizzle), as many as the tile has rows
//   warp 26     weight producer: one bulk copy of the packed 128 x 64 tile
//               (4 KB int4, 8 KB int8) and one of its scales
//   warp 17     allocates TMEM and issues tcgen05.mma (A from TMEM, B from
//               shared memory); producers and MMA run their loops as whole
//               warps and predicate each issue on one elected lane
//   warps 18-25 epilogue: TMEM -> registers (tcgen05.ld), scale / bias /
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
#include "tc_common.cuh"
#include "fp4_decode.cuh"

namespace qmoe {
namespace {

constexpr int kDeqWarps = 16;                            // two groups of 8, alternate stages
constexpr int kWarpProd = 16;
constexpr int kWarpMma = 17;
constexpr int kWarpEpi0 = 18;
constexpr int kEpiWarps = 8;
constexpr int kWarpProd2 = kWarpEpi0 + kEpiWarps;          // second producer (weights)
constexpr int kTcThreads = (kWarpProd2 + 1) * 32;           // 864
constexpr int kBK = 64;                                    // k per stage
constexpr int kAStageCols = kBK / 2;                       // TMEM columns of one A tile
constexpr int kScaleBytesMax = 4 * kTilesPerBlock * 16 * 4;  // 4 blocks of fp32 pairs

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

template <int BITS, bool PERCOL, int BNMAX, int STAGES, bool FP4>
__global__ void __launch_bounds__(kTcThreads, 1)
    ffn_tc_kernel(const __grid_constant__ CUtensorMap bmap, const TcArgs a) {
    using C = TcCfg<BITS, PERCOL, BNMAX, STAGES>;
    // stages a role tests at once: within one lap of the ring (a dequantise
    // group's own stages are every other one)
    constexpr int kLook = STAGES - 1 < 4 ? STAGES - 1 : 4;
    constexpr int kLookDeq = (STAGES - 1) / 2 + 1 < 4 ? (STAGES - 1) / 2 + 1 : 4;
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
            mbar_init(smem_u32(&full[s]), 2);  // one arrival per producer warp
            mbar_init(smem_u32(&deq[s]), kDeqWarps / 2);  // one group decodes a stage
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

    if (warp == kWarpProd || warp == kWarpProd2) {
        // ------------------------------------------------------- producers
        // warp kWarpProd: the activation boxes; warp kWarpProd2: the packed
        // codes and their scales. Each arrives once on the stage's full barrier
        // with its own byte count, so the two issue streams run side by side.
        const bool acts = warp == kWarpProd;
        const uint32_t e = elect_one();
        int st = 0;
        uint32_t ph = 0;
        bool ok = true;
        int ready = 0;  // free stages found ahead by the last batched test
        const int ngr = int(a.K / kgroup_of(BITS));
        const int bs_log2 = PERCOL ? 0 : __ffs(a.block_size) - 1;
        for (int i = blockIdx.x; ok && i < total; i += gridDim.x) {
            const Item it = item_at(i, prefix, a, nrb, nks);
            const int nbox = (it.rows + C::kBoxRows - 1) / C::kBoxRows;
            const uint32_t bytes = acts ? uint32_t(nbox * C::kBoxRows * 128) : uint32_t(C::kPacked) + sbytes;
            const int y0 = int(it.seg0) + it.tt * a.bn;
            const int64_t blk = int64_t(it.e) * nrb + it.rb;
            for (int ks = it.ks_lo; ks < it.ks_hi; ++ks) {
                if (ready == 0) {
                    ready = ready_run<kLook>(empty, nullptr, st, ph ^ 1u, 1, STAGES);
                    if (ready == 0) {
                        if (!warp_wait(smem_u32(&empty[st]), ph ^ 1u, abort_flag, a.status, a.timeout_ns)) { ok = false; break; }
                        ready = 1;
                    }
                }
                --ready;
                uint8_t* sb = smem + st * C::kStage;
                const uint32_t fb = smem_u32(&full[st]);
                mbar_expect_tx_e(fb, bytes, e);
                if (acts) {
                    for (int b = 0; b < nbox; ++b)
                        tma_2d_e(smem_u32(sb + b * C::kBoxRows * 128), &bmap, ks * kBK, y0 + b * C::kBoxRows, fb, e);
                } else {
                    const int g = ks * (kBK / kgroup_of(BITS));  // first k-group of the stage
                    const uint8_t* src = a.W + (blk * ngr + g) * int64_t(kTilesPerBlock) * kUnitBytes;
                    bulk_g2s_e(smem_u32(sb + C::kB), src, C::kPacked, fb, e);
                    if (!PERCOL) {
                        const int b0 = (ks * kBK) >> bs_log2;
                        const uint8_t* ssrc = reinterpret_cast<const uint8_t*>(a.S) +
                                              (blk * nsb + b0) * int64_t(kTilesPerBlock * 16 * ssz);
                        bulk_g2s_e(smem_u32(sb + C::kB + C::kPacked), ssrc, sbytes, fb, e);
                    }
                }
                if (++st == STAGES) { st = 0; ph ^= 1u; }
            }
        }
    } else if (warp == kWarpMma) {
        // ------------------------------------------------------- MMA issuer
        {
            const uint32_t e = elect_one();
            int st = 0, acc = 0;
            uint32_t ph = 0, aph = 0;
            bool ok = true;
            int ready = 0;  // decoded stages found ahead by the last batched test
            for (int i = blockIdx.x; ok && i < total; i += gridDim.x) {
                const Item it = item_at(i, prefix, a, nrb, nks);
                const int n = ((it.rows + 15) / 16) * 16;
                const uint32_t idesc = idesc_bf16(n);
                if (!warp_wait(smem_u32(&acce[acc]), aph ^ 1u, abort_flag, a.status, a.timeout_ns)) break;
                tc_fence_after();
                const uint32_t d = tmem + uint32_t(acc * BNMAX);
                for (int ks = it.ks_lo; ks < it.ks_hi; ++ks) {
                    // a stage is ready when decoded (A) and landed (B)
                    if (ready == 0) {
                        ready = ready_run<kLook>(deq, full, st, ph, 1, STAGES);
                        if (ready == 0) {
                            if (!warp_wait(smem_u32(&deq[st]), ph, abort_flag, a.status, a.timeout_ns) ||
                                !warp_wait(smem_u32(&full[st]), ph, abort_flag, a.status, a.timeout_ns)) { ok = false; break; }
                            ready = 1;
                        }
                    }
                    --ready;
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
                // test hook: with a.withhold the first item's accumulator is never
                // announced, so the epilogue's bounded wait runs out (no fault)
                mma_commit_e(smem_u32(&accf[acc]), (a.withhold && i == int(blockIdx.x)) ? 0u : e);
                if (++acc == 2) { acc = 0; aph ^= 1u; }
            }
        }
    } else if (warp < kDeqWarps) {
        // ------------------------------------------------------- dequantise
        // warp w writes row tile t = 2*(w%4) + (w/4)%2 (TMEM lanes 16t..16t+15,
        // inside the lane quarter w%4 it may access) of the stages of parity
        // w / 8: two groups of eight warps decode alternate stages
        const int tile = 2 * (warp & 3) + ((warp >> 2) & 1), grp = warp >> 3;
        const int r0 = lane >> 2, c = lane & 3;
        const uint32_t lane_addr = uint32_t(16 * tile) << 16;
        int st = 0;
        uint32_t ph = 0;
        bool ok = true;
        const uint32_t kMask = 0x000F000Fu, kMagic = 0x43004300u, kBias4 = 0x43084308u;
        // scale block (within the stage) of a k offset: blocks of 64 k or more
        // cover the whole stage
        const int bs_shift = a.block_size >= kBK ? 30 : __ffs(a.block_size) - 1;
        const bool stage_scale = a.block_size >= kBK;
        int ready = 0;  // this group's landed stages found ahead by the last batched test
        // The decode of a stage depends on nothing but its buffers, so the
        // group walks its own stages (every other one of the CTA's sequence)
        // directly: the stage count of the CTA's items, then a flat loop.
        int nstages = 0;
        for (int i = blockIdx.x; i < total; i += gridDim.x) {
            const Item it = item_at(i, prefix, a, nrb, nks);
            nstages += it.ks_hi - it.ks_lo;
        }
        if (grp == 1) st = 1;
        for (int n = grp; ok && n < nstages; n += 2) {
            {
                if (ready == 0) {
                    ready = ready_run<kLookDeq>(full, nullptr, st, ph, 2, STAGES);
                    if (ready == 0) {
                        if (!warp_wait(smem_u32(&full[st]), ph, abort_flag, a.status, a.timeout_ns)) { ok = false; break; }
                        ready = 1;
                    }
                }
                --ready;
                const uint8_t* sb = smem + st * C::kStage;
                const uint8_t* pk = sb + C::kB;
                const uint8_t* sc = pk + C::kPacked;
                const uint32_t at = tmem + lane_addr + uint32_t(C::kACol0 + st * kAStageCols);
                // bf16 scale of rows r0 / r0 + 8 (in both halves) of the block
                // holding stage-relative k offset kl
                auto scale_pair = [&](int kl, uint32_t& sa2, uint32_t& sb2) {
                    const int si = ((kl >> bs_shift) * kTilesPerBlock + tile) * 16 + 2 * r0;
                    if (a.scale_bf16) {
                        const uint32_t raw = *reinterpret_cast<const uint32_t*>(sc + si * 2);
                        sa2 = __byte_perm(raw, 0u, 0x1010);
                        sb2 = __byte_perm(raw, 0u, 0x3232);
                    } else {
                        const float2 f = *reinterpret_cast<const float2*>(sc + si * 4);
                        sa2 = bf2_bcast(f.x);
                        sb2 = bf2_bcast(f.y);
                    }
                };
                // blocks of 64 k or more: one scale pair for the whole stage
                uint32_t sa_st = 0, sb_st = 0;
                if (!PERCOL && stage_scale) scale_pair(0, sa_st, sb_st);
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
                        if (BITS == 4 && FP4) {
                            decode_fp4x8(wv[j], A);  // MXFP4: e2m1 values, no zero point
                        } else if (BITS == 4) {
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
                            uint32_t sa2 = sa_st, sb2 = sb_st;
                            if (!stage_scale) scale_pair(32 * gg * (BITS == 8) + 16 * j + 4 * c, sa2, sb2);
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
                st += 2;
                if (st >= STAGES) {
                    st -= STAGES;
                    ph ^= 1u;
                }
            }
        }
    } else if (warp >= kWarpEpi0 && warp < kWarpEpi0 + kEpiWarps) {
        // ------------------------------------------------------- epilogue
        const int qd = warp & 3;                        // TMEM lane quarter this warp may read
        const int half = (warp - kWarpEpi0) >> 2;       // which 16-column chunks it takes
        const int row = qd * 32 + lane;
        int acc = 0;
        uint32_t aph = 0;
        for (int i = blockIdx.x; i < total; i += gridDim.x) {
            const Item it = item_at(i, prefix, a, nrb, nks);
            if (!warp_wait(smem_u32(&accf[acc]), aph, abort_flag, a.status, a.timeout_ns)) break;
            tc_fence_after();
            tc_epilogue_item<PERCOL>(a, it, nrb, tmem + (uint32_t(qd * 32) << 16) + uint32_t(acc * BNMAX), row,
                                     lane, 16 * half, 32);
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

template <int BITS, bool PERCOL, int BNMAX, bool FP4>
struct Launch {
    static constexpr int kStage = TcCfg<BITS, PERCOL, BNMAX, 1>::kStage;
    static constexpr int kByTmem = (512 - 2 * BNMAX) / kAStageCols;
    static constexpr int kBySmem = (200 * 1024) / kStage;
    static constexpr int kStages = kByTmem < kBySmem ? (kByTmem < 12 ? kByTmem : 12) : (kBySmem < 12 ? kBySmem : 12);
    using C = TcCfg<BITS, PERCOL, BNMAX, kStages>;
    static cudaError_t prepare() {
        return cudaFuncSetAttribute(ffn_tc_kernel<BITS, PERCOL, BNMAX, kStages, FP4>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    }
    static cudaError_t run(const CUtensorMap& map, const TcArgs& a, int grid, cudaStream_t st) {
        ffn_tc_kernel<BITS, PERCOL, BNMAX, kStages, FP4><<<grid, kTcThreads, C::kSmem, st>>>(map, a);
        return cudaGetLastError();
    }
};

template <int BITS, bool PERCOL, bool FP4>
cudaError_t dispatch_bn(int bnmax, const CUtensorMap& map, const TcArgs& a, int grid, cudaStream_t st) {
    switch (bnmax) {
        case 16: return Launch<BITS, PERCOL, 16, FP4>::run(map, a, grid, st);
        case 32: return Launch<BITS, PERCOL, 32, FP4>::run(map, a, grid, st);
        case 64: return Launch<BITS, PERCOL, 64, FP4>::run(map, a, grid, st);
        default: return Launch<BITS, PERCOL, 128, FP4>::run(map, a, grid, st);
    }
}

template <int BITS, bool PERCOL, bool FP4>
cudaError_t prepare_bits() {
    cudaError_t e = Launch<BITS, PERCOL, 16, FP4>::prepare();
    if (e == cudaSuccess) e = Launch<BITS, PERCOL, 32, FP4>::prepare();
    if (e == cudaSuccess) e = Launch<BITS, PERCOL, 64, FP4>::prepare();
    if (e == cudaSuccess) e = Launch<BITS, PERCOL, 128, FP4>::prepare();
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


// Row p of the gathered activations is x[perm[p]] times the router weight
// of the (token, slot) pair at position p (found through inv), rounded once to
// the activation dtype. One thread per 16 bytes of output.
__global__ void gather_rows_weighted_kernel(const void* __restrict__ x, const int32_t* __restrict__ perm,
                                            const int32_t* __restrict__ inv, const float* __restrict__ topk_w,
                                            int k, void* __restrict__ xp, int64_t R, int64_t H, int act_bf16) {
    const int64_t per_vec = act_bf16 ? 8 : 4;
    const int64_t row_vecs = H / per_vec;
    const int64_t total = R * row_vecs;
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < total;
         i += int64_t(gridDim.x) * blockDim.x) {
        const int64_t p = i / row_vecs, v = i - p * row_vecs;
        const int64_t t = perm[p];
        float w = 0.0f;
        for (int j = 0; j < k; ++j)
            if (inv[t * k + j] == p) w = topk_w[t * k + j];
        const uint4 in = reinterpret_cast<const uint4*>(x)[t * row_vecs + v];
        uint4 out;
        if (act_bf16) {
            const uint32_t u[4] = {in.x, in.y, in.z, in.w};
            uint32_t r[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const __nv_bfloat162 b = __floats2bfloat162_rn(__uint_as_float(u[q] << 16) * w,
                                                               __uint_as_float(u[q] & 0xFFFF0000u) * w);
                r[q] = *reinterpret_cast<const uint32_t*>(&b);
            }
            out = make_uint4(r[0], r[1], r[2], r[3]);
        } else {
            out = make_uint4(__float_as_uint(__uint_as_float(in.x) * w), __float_as_uint(__uint_as_float(in.y) * w),
                             __float_as_uint(__uint_as_float(in.z) * w), __float_as_uint(__uint_as_float(in.w) * w));
        }
        reinterpret_cast<uint4*>(xp)[i] = out;
    }
}

}  // namespace

cudaError_t launch_gather_rows_weighted(const void* x, const int32_t* perm, const int32_t* inv,
                                        const float* topk_w, int k, void* xp, int64_t R, int64_t H, int act_bf16,
                                        cudaStream_t st) {
    if (R == 0) return cudaSuccess;
    const int64_t vecs = H / (act_bf16 ? 8 : 4);
    int64_t blocks = (R * vecs + 255) / 256;
    if (blocks > 148 * 8) blocks = 148 * 8;
    gather_rows_weighted_kernel<<<unsigned(blocks), 256, 0, st>>>(x, perm, inv, topk_w, k, xp, R, H, act_bf16);
    return cudaGetLastError();
}

cudaError_t prepare_ffn_tc() {
    cudaError_t e = prepare_bits<4, false, false>();
    if (e == cudaSuccess) e = prepare_bits<4, true, false>();
    if (e == cudaSuccess) e = prepare_bits<8, false, false>();
    if (e == cudaSuccess) e = prepare_bits<8, true, false>();
    if (e == cudaSuccess) e = prepare_bits<4, false, true>();  // MXFP4
    if (e == cudaSuccess) e = prepare_ffn_tc_decode();
    if (e == cudaSuccess) e = prepare_ffn_tc_wide();
    return e;
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
    if (bnmax > 128) return launch_ffn_tc_wide(f, bn, status, st);
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
    a.timeout_ns = f.timeout_ns;
    a.withhold = f.withhold;
    a.bn = bn;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const bool percol = f.block_size == 0;
    if (f.bits == 4)
        return f.fp4    ? dispatch_bn<4, false, true>(bnmax, map, a, sms, st)
               : percol ? dispatch_bn<4, true, false>(bnmax, map, a, sms, st)
                        : dispatch_bn<4, false, false>(bnmax, map, a, sms, st);
    return percol ? dispatch_bn<8, true, false>(bnmax, map, a, sms, st)
                  : dispatch_bn<8, false, false>(bnmax, map, a, sms, st);
}

}  // namespace qmoe
