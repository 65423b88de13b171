// ffn_tc_decode.cu -- expert FFN layers for few routed rows per expert on the
// tcgen05 tensor cores (sm_100a): a weight-streaming kernel.
//
// Each linear is y = x @ dequant(W).T + b ("QLinearWoQ" page, class summary)
// over the rows routed to one expert, with the packed weights decoded tile by
// tile inside the loop and never written out dense ("ClikaRT::nn::QMoEWoQ",
// class description). With at most 32 routed rows per expert the layer is
// bound by streaming the packed weights from HBM, so this kernel is organised
// around that stream:
//
//   * work items (expert, token tile, K split, 128-row block) are handed to
//     CTAs in contiguous runs, so consecutive items share their activations;
//     a run's activations ([tile rows x split's k range] bf16) arrive with one
//     3-D TMA and stay resident in shared memory;
//   * a stage is 128 k of one 128-row block: one bulk copy of the packed
//     codes (8 KB int4, 16 KB int8) into a ring that the dequantise warps
//     release as soon as they have read it, so the HBM stream never waits on
//     the tensor cores;
//   * 16 dequantise warps (two per 16-row tile, alternate stages) write the
//     exact centred codes q - z as bf16 straight into a ring of TMEM slots
//     (tcgen05.st); the MMA reads A from TMEM, B (activations) from shared
//     memory, and issues from a converged warp with the instruction
//     predicated on one elected lane;
//   * K-block scales are not multiplied into the weights: each stage's MMAs
//     write one fp32 partial sum per scale block into TMEM, and the epilogue
//     warps fold the partials into register accumulators as
//     acc += s_block * partial, reading the scales from a ring of their own
//     that the producer fills one stage at a time. Per-column scales
//     (block_size 0) accumulate the whole item in TMEM and scale once.
//
// Work per stage and tile is then: decode (shift, mask, OR, one bf16 subtract
// per two weights), eight 128 x N x 16 MMAs, and N fused multiply-adds per
// scale block in the epilogue. Every wait is bounded: after about two seconds
// the kernel records QMOE_TIMEOUT in the workspace status word, every role
// leaves its loop, and the CTA frees its TMEM and exits.
#include <algorithm>

#include "qmoe_internal.cuh"
#include "tc_common.cuh"
#include "fp4_decode.cuh"

namespace qmoe {
namespace {

constexpr int kDBK = 128;                 // k per stage
constexpr int kDAStageCols = kDBK / 2;    // TMEM columns of one decoded A tile
constexpr int kDDeqWarps = 16;            // warps 0-15 dequantise
constexpr int kDWarpProd = 16;            // producer
constexpr int kDWarpMma = 17;             // TMEM allocation and MMA issue
constexpr int kDEpi0 = 18;                // warps 18-21: epilogue
constexpr int kDEpiWarps = 4;
constexpr int kDThreads = (kDEpi0 + kDEpiWarps) * 32;  // 704

constexpr int kDRingMax = 8;              // packed-code ring slots at most
constexpr int kDSRingMax = 24;            // scale ring slots at most
constexpr int kDBMax = 128 * 1024;        // resident activations
constexpr int kDBarBytes = 3072;          // barriers, TMEM slot, item prefix
constexpr int kDPrefixOff = 768;          // item prefix sums inside the barrier area
constexpr int kDSmemMax = 227 * 1024;

// SMODE 0: per-column scales (one accumulator per item, scaled at the end);
// SMODE 1, 2, 4: that many scale blocks per 128-k stage (block size >= 128,
// 64, 32), one fp32 partial per block and stage.
template <int BITS, int SMODE, int BN>
struct TcdCfg {
    static constexpr int kPacked = kBlockRows * kDBK * BITS / 8;   // packed bytes of one stage
    static constexpr int kSP = SMODE == 0 ? 1 : SMODE;            // partials per stage
    static constexpr int kPC = kSP * BN;                           // TMEM columns per partial slot
    static constexpr int kPR = (SMODE == 0 || kPC >= 128) ? 2 : 4;  // partial slots
    static constexpr int kACol0 = kPR * kPC;
    static constexpr int kAS0 = (512 - kACol0) / kDAStageCols;
    static constexpr int kAS = kAS0 > 7 ? 7 : kAS0;                // A-tile slots
    static_assert(kAS >= 4, "TMEM budget");
    static_assert(kACol0 + kAS * kDAStageCols <= 512, "TMEM budget");
};

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

__device__ __forceinline__ bool same_run(const Item& p, const Item& q) {
    return p.e == q.e && p.tt == q.tt && p.split == q.split;
}

// Scale of packed row `row` (0..127 of the row block) inside one block of 128
// scales stored in pair order (r0, r0 + 8) per 16-row tile.
__device__ __forceinline__ int scale_pos(int row) {
    const int rr = row & 15;
    return (row >> 4) * 16 + (rr & 7) * 2 + (rr >> 3);
}

template <int BITS, int SMODE, int BN, bool FP4>
__global__ void __launch_bounds__(kDThreads, 1)
    ffn_tc_decode_kernel(const __grid_constant__ CUtensorMap bmap, const TcArgs a) {
    using C = TcdCfg<BITS, SMODE, BN>;
    constexpr int AS = C::kAS, PR = C::kPR, SP = C::kSP;
    const int PS = a.ring;          // packed-ring slots (>= 2)
    const int SR = a.sring;         // scale-ring slots (SMODE != 0)
    const int SSLOT = a.stage_bytes;  // bytes of one scale-ring slot
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint8_t* bsm = smem;                                   // activations [chunk][BN rows][128 B]
    uint8_t* bar_area = smem + kDBMax;
    uint8_t* psm = bar_area + kDBarBytes;                  // packed-code ring
    uint8_t* ssm = psm + PS * C::kPacked;                  // scale ring
    uint64_t* pfull = reinterpret_cast<uint64_t*>(bar_area);
    uint64_t* pempty = pfull + kDRingMax;
    uint64_t* afull = pempty + kDRingMax;
    uint64_t* aempty = afull + 8;
    uint64_t* cfull = aempty + 8;                          // partial (or accumulator) slot written
    uint64_t* cempty = cfull + 4;                          // ... and read by the epilogue
    uint64_t* sfull = cempty + 4;
    uint64_t* sempty = sfull + kDSRingMax;
    uint64_t* bfull = sempty + kDSRingMax;
    uint64_t* bempty = bfull + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bempty + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* prefix = reinterpret_cast<int*>(bar_area + kDPrefixOff);

    const int nrb = int(padded_rows(a.N) / kBlockRows);
    const int nks = int(a.K / kDBK);

    if (tid == 0) {
        for (int s = 0; s < PS; ++s) {
            mbar_init(smem_u32(&pfull[s]), 1);
            mbar_init(smem_u32(&pempty[s]), kDDeqWarps / 2);
        }
        for (int s = 0; s < AS; ++s) {
            mbar_init(smem_u32(&afull[s]), kDDeqWarps / 2);
            mbar_init(smem_u32(&aempty[s]), 1);
        }
        for (int s = 0; s < PR; ++s) {
            mbar_init(smem_u32(&cfull[s]), 1);
            mbar_init(smem_u32(&cempty[s]), kDEpiWarps);
        }
        for (int s = 0; s < SR; ++s) {
            mbar_init(smem_u32(&sfull[s]), 1);
            mbar_init(smem_u32(&sempty[s]), kDEpiWarps);
        }
        mbar_init(smem_u32(bfull), 1);
        mbar_init(smem_u32(bempty), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        // items per expert: token tiles x splits x row blocks; exclusive prefix
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
    // this CTA's contiguous range of items
    const int i_lo = int((int64_t(blockIdx.x) * total) / gridDim.x);
    const int i_hi = int((int64_t(blockIdx.x + 1) * total) / gridDim.x);
    const int ssz = a.scale_bf16 ? 2 : 4;
    const int nsb = SMODE == 0 ? 1 : int(a.K / a.block_size);

    if (warp == kDWarpProd) {
        // ------------------------------------------------------- producer
        const uint32_t e = elect_one();
        int ps = 0, ss = 0;
        uint32_t pph = 0, sph = 0, bph = 0;
        bool ok = true;
        const int ngr = int(a.K / kgroup_of(BITS));
        const int bs_log2 = SMODE == 0 ? 0 : __ffs(a.block_size) - 1;
        const uint8_t* sbase = static_cast<const uint8_t*>(a.S);
        Item prev{};
        prev.e = -1;
        for (int i = i_lo; ok && i < i_hi; ++i) {
            const Item it = item_at_stream(i, prefix, a, nrb, nks);
            if (prev.e < 0 || !same_run(prev, it)) {
                // the run's activations: rows [seg0 + tt*bn, +BN), 64-k chunks from
                // ks_lo*2; the box spans the largest split (out-of-range rows and
                // chunks arrive as zeros)
                if (!warp_wait(smem_u32(bempty), bph ^ 1u, abort_flag, a.status, a.timeout_ns)) { ok = false; break; }
                bph ^= 1u;
                const int box_ch = ((nks + a.splits - 1) / a.splits) * (kDBK / 64);
                mbar_expect_tx_e(smem_u32(bfull), uint32_t(box_ch * BN * 128), e);
                tma_3d_e(smem_u32(bsm), &bmap, 0, int(it.seg0) + it.tt * a.bn, it.ks_lo * (kDBK / 64),
                         smem_u32(bfull), e);
            }
            prev = it;
            const int64_t blk = int64_t(it.e) * nrb + it.rb;
            for (int ks = it.ks_lo; ks < it.ks_hi; ++ks) {
                if (!warp_wait(smem_u32(&pempty[ps]), pph ^ 1u, abort_flag, a.status, a.timeout_ns)) { ok = false; break; }
                const uint32_t fb = smem_u32(&pfull[ps]);
                mbar_expect_tx_e(fb, uint32_t(C::kPacked), e);
                const int g = ks * (kDBK / kgroup_of(BITS));
                const uint8_t* src = a.W + (blk * ngr + g) * int64_t(kTilesPerBlock) * kUnitBytes;
                bulk_g2s_e(smem_u32(psm + ps * C::kPacked), src, C::kPacked, fb, e);
                if (++ps == PS) { ps = 0; pph ^= 1u; }
                if (SMODE != 0) {
                    // the stage's scale blocks [sb0, sb0 + SP): contiguous, 128 scales each
                    if (!warp_wait(smem_u32(&sempty[ss]), sph ^ 1u, abort_flag, a.status, a.timeout_ns)) { ok = false; break; }
                    const uint32_t sb = smem_u32(&sfull[ss]);
                    mbar_expect_tx_e(sb, uint32_t(SSLOT), e);
                    const int sb0 = (ks * kDBK) >> bs_log2;
                    const uint8_t* ssrc = sbase + (blk * nsb + sb0) * (kBlockRows * ssz);
                    bulk_g2s_e(smem_u32(ssm + ss * SSLOT), ssrc, uint32_t(SSLOT), sb, e);
                    if (++ss == SR) { ss = 0; sph ^= 1u; }
                }
            }
        }
    } else if (warp == kDWarpMma) {
        // ------------------------------------------------------- MMA issue
        const uint32_t e = elect_one();
        int as = 0, pr = 0;
        uint32_t aph = 0, cph = 0, bph = 0;
        bool ok = true;
        Item prev{};
        prev.e = -1;
        const uint32_t b0 = smem_u32(bsm);
        for (int i = i_lo; ok && i < i_hi; ++i) {
            const Item it = item_at_stream(i, prefix, a, nrb, nks);
            if (prev.e < 0 || !same_run(prev, it)) {
                if (!warp_wait(smem_u32(bfull), bph, abort_flag, a.status, a.timeout_ns)) break;
                bph ^= 1u;
            }
            prev = it;
            const uint32_t idesc = idesc_bf16(((it.rows + 15) / 16) * 16);
            if (SMODE == 0) {
                // one accumulator slot for the whole item
                if (!warp_wait(smem_u32(&cempty[pr]), cph ^ 1u, abort_flag, a.status, a.timeout_ns)) break;
                tc_fence_after();
            }
            for (int ks = it.ks_lo; ks < it.ks_hi; ++ks) {
                // with per-stage partials, a full A slot also means a free partial
                // slot: the dequantise warps waited for it before signalling
                if (!warp_wait(smem_u32(&afull[as]), aph, abort_flag, a.status, a.timeout_ns)) { ok = false; break; }
                tc_fence_after();
                const uint32_t at = tmem + uint32_t(C::kACol0 + as * kDAStageCols);
                const uint32_t d0 = tmem + uint32_t(pr * C::kPC);
                // this stage's first 64-k chunk of the resident activations
                const uint64_t bd = desc_sw128(b0 + uint32_t((ks - it.ks_lo) * (kDBK / 64) * BN * 128));
                const uint32_t first = (SMODE == 0 && ks > it.ks_lo) ? 1u : 0u;
#pragma unroll
                for (int kk = 0; kk < kDBK / 16; ++kk) {
                    // chunk kk/4 (BN rows of 128 B), 32 B per 16 k inside the swizzled row
                    const uint64_t bk = bd + uint64_t(((kk / 4) * BN * 128 + 32 * (kk % 4)) >> 4);
                    constexpr int kPerPart = (kDBK / 16) / SP;  // MMAs per scale block
                    const uint32_t d = SMODE == 0 ? d0 : d0 + uint32_t((kk / kPerPart) * BN);
                    const uint32_t accum = SMODE == 0 ? (kk > 0 ? 1u : first) : (kk % kPerPart ? 1u : 0u);
                    mma_bf16_ts_e(d, at + uint32_t(8 * kk), bk, idesc, accum, e);
                }
                mma_commit_e(smem_u32(&aempty[as]), e);
                if (++as == AS) { as = 0; aph ^= 1u; }
                if (SMODE != 0) {
                    mma_commit_e(smem_u32(&cfull[pr]), e);
                    if (++pr == PR) { pr = 0; cph ^= 1u; }
                }
            }
            if (!ok) break;
            if (SMODE == 0) {
                mma_commit_e(smem_u32(&cfull[pr]), e);
                if (++pr == PR) { pr = 0; cph ^= 1u; }
            }
            // release the resident activations after the run's last item
            bool last = i + 1 >= i_hi;
            if (!last) last = !same_run(it, item_at_stream(i + 1, prefix, a, nrb, nks));
            if (last) mma_commit_e(smem_u32(bempty), e);
        }
    } else if (warp < kDDeqWarps) {
        // ------------------------------------------------------- dequantise
        // tile: TMEM lanes 16*tile.. lie in this warp's lane quarter (warp % 4);
        // par: this warp takes the stages of that parity (stage count in the CTA)
        const int tile = 2 * (warp & 3) + ((warp >> 2) & 1);
        const int par = warp >> 3;
        const uint32_t lane_addr = uint32_t(16 * tile) << 16;
        int ps = par, as = par;  // both rings have at least two slots
        uint32_t pph = 0, aph = 0;
        int sn = 0;
        bool ok = true;
        const uint32_t kMask = 0x000F000Fu, kMagic = 0x43004300u, kBias4 = 0x43084308u;
        constexpr int GROUPS = kDBK / kgroup_of(BITS);  // 2 (int4) or 4 (int8)
        constexpr int KSTEPS = kgroup_of(BITS) / 16;
        for (int i = i_lo; ok && i < i_hi; ++i) {
            const Item it = item_at_stream(i, prefix, a, nrb, nks);
            for (int ks = it.ks_lo; ks < it.ks_hi; ++ks) {
                if (((sn++) & 1) != par) continue;
                if (!warp_wait(smem_u32(&pfull[ps]), pph, abort_flag, a.status, a.timeout_ns)) { ok = false; break; }
                uint4 wq[GROUPS];
                const uint8_t* pk = psm + ps * C::kPacked;
#pragma unroll
                for (int gg = 0; gg < GROUPS; ++gg)
                    wq[gg] = *reinterpret_cast<const uint4*>(pk + ((gg * kTilesPerBlock + tile) * 32 + lane) * 16);
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&pempty[ps]));
                ps += 2;
                if (ps >= PS) { ps -= PS; pph ^= 1u; }
                if (!warp_wait(smem_u32(&aempty[as]), aph ^ 1u, abort_flag, a.status, a.timeout_ns)) { ok = false; break; }
                tc_fence_after();
                const uint32_t at = tmem + lane_addr + uint32_t(C::kACol0 + as * kDAStageCols);
#pragma unroll
                for (int gg = 0; gg < GROUPS; ++gg) {
                    const uint32_t wv[4] = {wq[gg].x, wq[gg].y, wq[gg].z, wq[gg].w};
                    uint32_t r[4 * KSTEPS];
#pragma unroll
                    for (int j = 0; j < KSTEPS; ++j) {
                        uint32_t A[4];  // (r0, k 0-1), (r0+8, k 0-1), (r0, k 2-3), (r0+8, k 2-3)
                        if (BITS == 4 && FP4) {
                            decode_fp4x8(wv[j], A);  // MXFP4: e2m1 values, no zero point
                        } else if (BITS == 4) {
                            // nibble q OR bf16 128.0 is 128 + q exactly; minus 136.0 gives q - 8
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
                        // 16x256b fragment: (r0, col 2c), (r0, col 2c+1), (r0+8, col 2c), (r0+8, col 2c+1)
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
                if (SMODE != 0) {
                    // the stage's partial slot must have been read by the epilogue
                    // (stage s uses slot s % PR, phase (s / PR) & 1), so the MMA
                    // needs only this one barrier
                    const int s = sn - 1;
                    if (!warp_wait(smem_u32(&cempty[s % PR]), ((s / PR) & 1) ^ 1u, abort_flag, a.status, a.timeout_ns)) {
                        ok = false;
                        break;
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&afull[as]));
                as += 2;
                if (as >= AS) { as -= AS; aph ^= 1u; }
            }
        }
    } else {
        // ------------------------------------------------------- epilogue
        // warp w reads TMEM lane quarter w % 4: packed row qd*32 + lane
        const int qd = warp & 3;
        const int row = qd * 32 + lane;
        const uint32_t lane_base = tmem + (uint32_t(qd * 32) << 16);
        const int spos = scale_pos(row);
        int pr = 0, ss = 0;
        uint32_t cph = 0, sph = 0;
        bool ok = true;
        for (int i = i_lo; ok && i < i_hi; ++i) {
            const Item it = item_at_stream(i, prefix, a, nrb, nks);
            const int64_t prow = int64_t(it.rb) * kBlockRows + row;  // packed row in the expert
            const bool valid = prow < a.N;
            float acc[BN];
#pragma unroll
            for (int n = 0; n < BN; ++n) acc[n] = 0.0f;
            if (SMODE == 0) {
                if (!warp_wait(smem_u32(&cfull[pr]), cph, abort_flag, a.status, a.timeout_ns)) break;
                tc_fence_after();
                const int64_t si = (int64_t(it.e) * nrb + it.rb) * kBlockRows + spos;
                const float s = !valid ? 0.0f
                                : a.scale_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(a.S)[si])
                                               : reinterpret_cast<const float*>(a.S)[si];
                const bool empty_k = it.ks_hi <= it.ks_lo;  // no MMA wrote the accumulator
#pragma unroll
                for (int c0 = 0; c0 < BN; c0 += 16) {
                    float v[16];
                    tmem_ld16(lane_base + uint32_t(pr * C::kPC + c0), v);
#pragma unroll
                    for (int j = 0; j < 16; ++j) acc[c0 + j] = empty_k ? 0.0f : v[j] * s;
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&cempty[pr]));
                if (++pr == PR) { pr = 0; cph ^= 1u; }
            } else {
                for (int ks = it.ks_lo; ks < it.ks_hi; ++ks) {
                    if (!warp_wait(smem_u32(&sfull[ss]), sph, abort_flag, a.status, a.timeout_ns) ||
                        !warp_wait(smem_u32(&cfull[pr]), cph, abort_flag, a.status, a.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint8_t* sc = ssm + ss * SSLOT;
#pragma unroll
                    for (int q = 0; q < SP; ++q) {
                        const float s = a.scale_bf16
                                            ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(sc)[q * 128 + spos])
                                            : reinterpret_cast<const float*>(sc)[q * 128 + spos];
#pragma unroll
                        for (int c0 = 0; c0 < BN; c0 += 16) {
                            float v[16];
                            tmem_ld16(lane_base + uint32_t(pr * C::kPC + q * BN + c0), v);
#pragma unroll
                            for (int j = 0; j < 16; ++j) acc[c0 + j] = fmaf(v[j], s, acc[c0 + j]);
                        }
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive(smem_u32(&cempty[pr]));
                        mbar_arrive(smem_u32(&sempty[ss]));
                    }
                    if (++pr == PR) { pr = 0; cph ^= 1u; }
                    if (++ss == SR) { ss = 0; sph ^= 1u; }
                }
                if (!ok) break;
            }
            const float bias = (a.bias && valid) ? a.bias[int64_t(it.e) * a.N + prow] : 0.0f;
#pragma unroll
            for (int col = 0; col < BN; ++col) {
                const float val = acc[col] + bias;
                const bool in = col < it.rows;
                const int64_t p = it.seg0 + int64_t(it.tt) * a.bn + col;  // permuted row
                if (a.is_fc1) {
                    if (a.gated) {
                        // tile rows 0-7 are gate rows, 8-15 the matching up rows
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
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kDWarpMma) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
    }
}

template <int BITS, int SMODE, int BN, bool FP4>
struct LaunchD {
    static cudaError_t prepare() {
        return cudaFuncSetAttribute(ffn_tc_decode_kernel<BITS, SMODE, BN, FP4>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, kDSmemMax);
    }
    static cudaError_t run(const CUtensorMap& map, const TcArgs& a, int grid, cudaStream_t st) {
        const int smem = 1024 + kDBMax + kDBarBytes + a.ring * TcdCfg<BITS, SMODE, BN>::kPacked +
                         a.sring * a.stage_bytes;
        ffn_tc_decode_kernel<BITS, SMODE, BN, FP4><<<grid, kDThreads, smem, st>>>(map, a);
        return cudaGetLastError();
    }
};

template <int BITS, int SMODE, bool FP4>
cudaError_t prepare_mode() {
    cudaError_t e = LaunchD<BITS, SMODE, 16, FP4>::prepare();
    if (e == cudaSuccess) e = LaunchD<BITS, SMODE, 32, FP4>::prepare();
    return e;
}

template <int BITS, int SMODE, bool FP4>
cudaError_t run_mode(int bn, const CUtensorMap& map, const TcArgs& a, int grid, cudaStream_t st) {
    return bn <= 16 ? LaunchD<BITS, SMODE, 16, FP4>::run(map, a, grid, st) : LaunchD<BITS, SMODE, 32, FP4>::run(map, a, grid, st);
}

template <int BITS, bool FP4>
cudaError_t run_bits(int smode, int bn, const CUtensorMap& map, const TcArgs& a, int grid, cudaStream_t st) {
    switch (smode) {
        case 0: return run_mode<BITS, 0, FP4>(bn, map, a, grid, st);
        case 1: return run_mode<BITS, 1, FP4>(bn, map, a, grid, st);
        case 2: return run_mode<BITS, 2, FP4>(bn, map, a, grid, st);
        default: return run_mode<BITS, 4, FP4>(bn, map, a, grid, st);
    }
}

// Scale blocks per 128-k stage (0: per-column scales); -1 if unsupported.
int smode_of(int block_size) {
    if (block_size == 0) return 0;
    if (block_size >= kDBK) return 1;
    if (block_size == 64) return 2;
    if (block_size == 32) return 4;
    return -1;
}

}  // namespace

cudaError_t prepare_ffn_tc_decode() {
    cudaError_t e = cudaSuccess;
    if (e == cudaSuccess) e = prepare_mode<4, 0, false>();
    if (e == cudaSuccess) e = prepare_mode<4, 1, false>();
    if (e == cudaSuccess) e = prepare_mode<4, 2, false>();
    if (e == cudaSuccess) e = prepare_mode<4, 4, false>();
    if (e == cudaSuccess) e = prepare_mode<8, 0, false>();
    if (e == cudaSuccess) e = prepare_mode<8, 1, false>();
    if (e == cudaSuccess) e = prepare_mode<8, 2, false>();
    if (e == cudaSuccess) e = prepare_mode<8, 4, false>();
    if (e == cudaSuccess) e = prepare_mode<4, 4, true>();  // MXFP4 (block 32: four blocks per stage)
    return e;
}

bool tc_decode_fits(int64_t K, int splits, int bn, int block_size) {
    if (K % kDBK != 0 || bn > 32 || splits < 1 || smode_of(block_size) < 0) return false;
    const int64_t nks = K / kDBK;
    const int64_t per = (nks + splits - 1) / splits;  // largest split, in stages
    const int bnr = bn <= 16 ? 16 : 32;
    return per * kDBK * 2 * bnr <= kDBMax;
}

cudaError_t launch_ffn_tc_decode(const FfnArgs& f, int bn, int32_t* status, cudaStream_t st) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    const int bnr = bn <= 16 ? 16 : 32;
    const int smode = smode_of(f.block_size);
    if (!tc_decode_fits(f.K, f.splits, bn, f.block_size) || f.E + 1 > (kDBarBytes - kDPrefixOff) / 4)
        return cudaErrorInvalidValue;
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
    a.timeout_ns = f.timeout_ns;
    a.withhold = f.withhold;
    a.bn = bn;
    // packed ring: 8 slots (int4) / 4 (int8), 64 KB either way; the scale ring
    // takes what is left, up to 24 stages (one slot per stage)
    const int packed = kBlockRows * kDBK * f.bits / 8;
    a.ring = f.bits == 4 ? kDRingMax : 4;
    const int ssz = f.scale_bf16 ? 2 : 4;
    a.stage_bytes = smode == 0 ? 0 : smode * kBlockRows * ssz;
    const int room = kDSmemMax - 1024 - kDBMax - kDBarBytes - a.ring * packed;
    a.sring = smode == 0 ? 0 : std::min(kDSRingMax, room / a.stage_bytes);
    if (smode != 0 && a.sring < 2) return cudaErrorInvalidValue;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (f.fp4) return run_mode<4, 4, true>(bn, map, a, sms, st);  // block 32
    return f.bits == 4 ? run_bits<4, false>(smode, bn, map, a, sms, st) : run_bits<8, false>(smode, bn, map, a, sms, st);
}

}  // namespace qmoe
