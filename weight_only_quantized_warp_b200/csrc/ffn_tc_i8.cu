// ffn_tc_i8.cu -- the int8 block compute tier of the expert FFN layers on the
// 5th-generation tensor cores (tcgen05.mma kind::i8), sm_100a.
//
// "ClikaRT::nn::QMoEWoQ" (class description): a packed block weight on the
// int8 block tier takes its activation rounded to per-block int8 before the
// dot, and the dot of one weight row is the sum over the K blocks of
//   s_w * s_x * sum_k (c_k - z) q_k
// (c the stored code, z = 2^(bits-1) its zero point, q the activation code,
// s_w and s_x the two block scales). The integer dot of every block is exact
// here: the weight codes become signed bytes c - z in tensor memory, the
// activation codes are signed bytes, and the MMA accumulates int32. The two
// scales differ from block to block, so each block's int32 partial is taken
// out of tensor memory and folded into fp32 registers:
//   acc[m][n] += float(P_b[m][n]) * (s_w[m][b] * s_x[n][b]).
//
// Operand roles as in the bf16 grouped GEMM: MMA M = 128 weight rows of one
// expert, N = the expert's token tile (16..64), K = 32 per instruction.
// Warps of one persistent CTA (736 threads, one CTA per SM):
//   warps 0-3    convert: packed codes (shared) -> signed bytes written into
//                tensor memory (tcgen05.st), the two 16-row tiles of the
//                warp's TMEM lane quarter
//   warp 4       activation producer: 64-row TMA boxes of the activation
//                codes, 128 codes (one 128-byte swizzled row) per token
//   warp 5       weight producer: one bulk copy of the stage's packed codes
//   warp 6       allocates TMEM, issues tcgen05.mma (A from TMEM, B from
//                shared memory), one int32 partial per K block, cycling
//                through four partial buffers
//   warps 7-22   fold each block's partial into fp32 registers (four warps
//                per TMEM lane quarter, 16-column chunks), then run the
//                epilogue (bias, activation, store) from tensor memory
// Stages of 128 k cycle through an S-deep ring (full: copies landed; deq: A
// written; empty: the MMAs reading the stage are done); the four partial
// buffers through pfull (the block's MMAs are done) and pempty (folded), so
// the MMAs run up to three blocks ahead of the fold. Every wait is
// bounded as in the bf16 kernels.
//
// Layouts. The converter lane (r0 = L/4, c = L%4) holds rows r0 and r0 + 8 at
// k = 16j + 4c + {0..3} of k-step j (the packed fragment order). A
// 16x256b tensor-memory store of a 32-k chunk (k-steps 2m, 2m + 1) puts its
// k-step 2m quad in column 2c and its k-step 2m + 1 quad in column 2c + 1, so
// the MMA's k position 4p + i of the chunk holds the code at
// k = 16 (p & 1) + 4 (p >> 1) + sigma(i), with sigma the byte order of the
// codes inside the quad (k + {0, 2, 1, 3} for 4-bit codes, which keep one row
// in the low and the other in the high nibbles of a word; natural for 8-bit
// codes). quantize_rows_i8_kernel writes the activation codes in exactly that
// order (layouts 2 and 3), so both operands pair the same k.
#include <cuda.h>

#include <type_traits>

#include "qmoe_internal.cuh"
#include "tc_common.cuh"

namespace qmoe {
namespace {

constexpr int kIConvWarps = 4;
constexpr int kIWarpProdA = 4;
constexpr int kIWarpProdW = 5;
constexpr int kIWarpMma = 6;
constexpr int kIFold0 = 7;
constexpr int kIFoldWarps = 16;
constexpr int kIThreads = (kIFold0 + kIFoldWarps) * 32;  // 736: 88 registers a thread
constexpr int kIBK = 128;                                  // k per stage
constexpr int kIACols = kIBK / 4;                          // TMEM columns of one A tile (4 codes each)

// the tensor-core kernels' arguments plus the activation block scales
// [rows, K / block_size] that the fold multiplies in
struct TcI8Args : TcArgs {
    const float* xs;
};

template <int BITS, int BNMAX, int STAGES>
struct I8Cfg {
    static constexpr int kBoxRows = BNMAX < 64 ? BNMAX : 64;      // rows of one activation TMA box
    static constexpr int kPacked = kBlockRows * kIBK * BITS / 8;  // 8 KB (4-bit) or 16 KB (8-bit)
    static constexpr int kB = BNMAX * kIBK;                       // activation codes: 128 B per token
    static constexpr int kStage = kB + kPacked;                   // multiple of 1024
    static constexpr int kNPB = 4;                                // int32 partial buffers
    static constexpr int kACol0 = kNPB * BNMAX;                   // A tiles after the partial buffers
    static_assert(kACol0 + STAGES * kIACols <= 512, "TMEM budget");
    static constexpr int kBarOff = STAGES * kStage;
    // after the barriers and the prefix table: the fold warps' scale scratch
    static constexpr int kScratchOff = 2048;
    // barriers, prefix table, scratch, alignment slack; at least 120 KB so one CTA per SM
    static constexpr int kSmemUse = kBarOff + kScratchOff + 16 * 16 * 4 + 1024;
    static constexpr int kSmem = kSmemUse > 120 * 1024 ? kSmemUse : 120 * 1024;
};

// Instruction descriptor: kind::i8, signed A and B (K-major), int32 D, M = 128.
__device__ __forceinline__ uint32_t idesc_s8(int n) {
    return (2u << 4) | (1u << 7) | (1u << 10) | (uint32_t(n >> 3) << 17) | (uint32_t(128 >> 4) << 24);
}

__device__ __forceinline__ void mma_s8_ts_e(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate, uint32_t e) {
    asm volatile(
        "{\n.reg .pred p, q;\nsetp.ne.b32 p, %4, 0;\nsetp.ne.b32 q, %5, 0;\n"
        "@q tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n}" ::"r"(tmem_d),
        "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(e));
}

__device__ __forceinline__ void tmem_ld16_u32(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld8_u32(uint32_t taddr, uint32_t (&r)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_st16_f32(uint32_t taddr, const float (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
        "%15,%16};" ::"r"(taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15]))
        : "memory");
}

__device__ __forceinline__ void tmem_st16x256_x1(uint32_t taddr, const uint32_t (&r)[4]) {
    asm volatile("tcgen05.st.sync.aligned.16x256b.x1.b32 [%0], {%1,%2,%3,%4};" ::"r"(taddr), "r"(r[0]),
                 "r"(r[1]), "r"(r[2]), "r"(r[3])
                 : "memory");
}

// An int32 block partial as fp32, exactly: |P| <= block_size * 128 * 127
// stays below 2^22 for blocks up to 256 codes, and adding 1.5 * 2^23 to such
// an integer lands in the binade [2^23, 2^24) whose unit is 1, so the integer
// add on the bit pattern and one fp32 subtraction convert it (two full-rate
// instructions instead of the slower int-to-float conversion); longer blocks
// take the conversion instruction.
template <bool SHORT_BLOCKS>
__device__ __forceinline__ float i32_to_f32_t(uint32_t p) {
    if (SHORT_BLOCKS) return __uint_as_float(p + 0x4B400000u) - 12582912.0f;
    return float(int32_t(p));
}

// Four 4-bit codes (one per byte, in bits 0-3) -> four signed bytes c - 8:
// flipping bit 3 gives c - 8 for c >= 8 and c + 8 = (c - 8) + 16 otherwise,
// whose byte then needs bits 4-7 set; (t & 8) * 30 is 0xF0 exactly there.
__device__ __forceinline__ uint32_t nib4_to_s8(uint32_t nib) {
    const uint32_t t = nib ^ 0x08080808u;
    return t | ((t & 0x08080808u) * 30u);
}

template <int BITS, int BNMAX, int STAGES>
__global__ void __launch_bounds__(kIThreads, 1)
    ffn_tc_i8_kernel(const __grid_constant__ CUtensorMap amap, const TcI8Args a) {
    using C = I8Cfg<BITS, BNMAX, STAGES>;
    constexpr int KG = kgroup_of(BITS);
    constexpr int kLook = STAGES - 1 < 4 ? STAGES - 1 : 4;  // stages a role tests at once
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    uint8_t* bar_area = smem + C::kBarOff;
    uint64_t* full = reinterpret_cast<uint64_t*>(bar_area);
    uint64_t* deq = full + STAGES;
    uint64_t* empty = deq + STAGES;
    uint64_t* pfull = empty + STAGES;
    uint64_t* pempty = pfull + C::kNPB;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(pempty + C::kNPB);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* prefix = reinterpret_cast<int*>(tmem_slot + 4);  // [E + 1]

    const int nrb = int(padded_rows(a.N) / kBlockRows);
    const int nks = int((a.K + kIBK - 1) / kIBK);
    const int nsb = int(a.K / a.block_size);

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&full[s]), 2);  // one arrival per producer warp
            mbar_init(smem_u32(&deq[s]), kIConvWarps);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        for (int b = 0; b < C::kNPB; ++b) {
            mbar_init(smem_u32(&pfull[b]), 1);
            mbar_init(smem_u32(&pempty[b]), kIFoldWarps);
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
    if (warp == kIWarpMma) {
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
    // k of the items' ranges: whole K blocks (the planner keeps K splits on
    // block boundaries), so a block never straddles two items
    auto k_lo = [&](const Item& it) { return it.ks_lo * kIBK; };
    auto k_hi = [&](const Item& it) { return min(int(a.K), it.ks_hi * kIBK); };

    if (warp == kIWarpProdA || warp == kIWarpProdW) {
        // ------------------------------------------------------- producers
        // warp kIWarpProdA: the activation-code boxes (128 codes wide; past K
        // the box reads zeros); warp kIWarpProdW: the packed weight codes of
        // the stage's k range. Each arrives once on the stage's full barrier
        // with its own byte count.
        const bool acts = warp == kIWarpProdA;
        const uint32_t e = elect_one();
        int st = 0;
        uint32_t ph = 0;
        bool ok = true;
        int ready = 0;  // free stages found ahead by the last batched test
        const int ngr = int(a.K / KG);
        for (int i = blockIdx.x; ok && i < total; i += gridDim.x) {
            const Item it = item_at(i, prefix, a, nrb, nks);
            const int nbox = (it.rows + C::kBoxRows - 1) / C::kBoxRows;
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
                const int kv = min(kIBK, int(a.K) - ks * kIBK);  // 128, or 64 at the end of K
                if (acts) {
                    mbar_expect_tx_e(fb, uint32_t(nbox * C::kBoxRows * 128), e);
                    for (int b = 0; b < nbox; ++b)
                        tma_2d_e(smem_u32(sb + b * C::kBoxRows * 128), &amap, ks * kIBK, y0 + b * C::kBoxRows, fb, e);
                } else {
                    const uint32_t pbytes = uint32_t(kv / KG) * kTilesPerBlock * kUnitBytes;
                    mbar_expect_tx_e(fb, pbytes, e);
                    const int g = ks * (kIBK / KG);  // first k-group of the stage
                    const uint8_t* src = a.W + (blk * ngr + g) * int64_t(kTilesPerBlock) * kUnitBytes;
                    bulk_g2s_e(smem_u32(sb + C::kB), src, pbytes, fb, e);
                }
                if (++st == STAGES) { st = 0; ph ^= 1u; }
            }
        }
    } else if (warp == kIWarpMma) {
        // ------------------------------------------------------- MMA issuer
        // One int32 partial per K block: the first MMA of a block waits for
        // its partial buffer to be folded and overwrites it; the block's last
        // MMA is followed by a commit to pfull.
        const uint32_t e = elect_one();
        int st = 0, pb = 0;
        uint32_t ph = 0, pph = 0;
        bool ok = true;
        int ready = 0;  // decoded stages found ahead by the last batched test
        const int mpb = a.block_size / 32;  // MMAs (32 k each) per K block
        bool committed = false;             // any partial announced yet
        int pfree = 0;                      // folded partial buffers found ahead
        for (int i = blockIdx.x; ok && i < total; i += gridDim.x) {
            const Item it = item_at(i, prefix, a, nrb, nks);
            const uint32_t idesc = idesc_s8(((it.rows + 15) / 16) * 16);
            int mb = 0;  // MMAs of the current K block issued so far (32 k each)
            for (int ks = it.ks_lo; ok && ks < it.ks_hi; ++ks) {
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
                const uint32_t at = tmem + uint32_t(C::kACol0 + st * kIACols);
                const uint64_t bd = desc_sw128(smem_u32(smem + st * C::kStage));
                const int nk = min(kIBK, int(a.K) - ks * kIBK) / 32;
                for (int kk = 0; kk < nk; ++kk) {
                    const bool first = mb == 0;
                    if (first) {
                        if (pfree == 0) {
                            pfree = ready_run<C::kNPB - 1>(pempty, nullptr, pb, pph ^ 1u, 1, C::kNPB);
                            if (pfree == 0) {
                                if (!warp_wait(smem_u32(&pempty[pb]), pph ^ 1u, abort_flag, a.status, a.timeout_ns)) { ok = false; break; }
                                pfree = 1;
                            }
                        }
                        --pfree;
                        tc_fence_after();
                    }
                    // 32 k per MMA: 8 A columns, 32 B into each swizzled row of B
                    mma_s8_ts_e(tmem + uint32_t(pb * BNMAX), at + uint32_t(8 * kk), bd + uint64_t(2 * kk), idesc,
                                first ? 0u : 1u, e);
                    if (++mb == mpb) {  // the block is complete
                        mb = 0;
                        // test hook: with a.withhold the item's first partial is never
                        // announced, so the fold warps' bounded wait runs out (no fault)
                        const bool hold = a.withhold && !committed;
                        committed = true;
                        mma_commit_e(smem_u32(&pfull[pb]), hold ? 0u : e);
                        if (++pb == C::kNPB) { pb = 0; pph ^= 1u; }
                    }
                }
                if (!ok) break;
                mma_commit_e(smem_u32(&empty[st]), e);
                if (++st == STAGES) { st = 0; ph ^= 1u; }
            }
        }
    } else if (warp < kIConvWarps) {
        // ------------------------------------------------------- convert
        // warp w writes row tiles 2w and 2w + 1 (TMEM lanes 32w..32w+31, the
        // lane quarter it may access) of every stage
        int st = 0;
        uint32_t ph = 0;
        bool ok = true;
        int ready = 0;  // landed stages found ahead by the last batched test
        int nstages = 0;
        for (int i = blockIdx.x; i < total; i += gridDim.x) {
            const Item it = item_at(i, prefix, a, nrb, nks);
            nstages += it.ks_hi - it.ks_lo;
        }
        // the stage's k extent, from the item sequence (128, or 64 at the end of K)
        int item = blockIdx.x, ks = 0, ks_hi = 0;
        for (int n = 0; ok && n < nstages; ++n) {
            while (ks >= ks_hi) {
                const Item it = item_at(item, prefix, a, nrb, nks);
                ks = it.ks_lo;
                ks_hi = it.ks_hi;
                item += gridDim.x;
            }
            const int ngs = min(kIBK, int(a.K) - ks * kIBK) / KG;
            ++ks;
            if (ready == 0) {
                ready = ready_run<kLook>(full, nullptr, st, ph, 1, STAGES);
                if (ready == 0) {
                    if (!warp_wait(smem_u32(&full[st]), ph, abort_flag, a.status, a.timeout_ns)) { ok = false; break; }
                    ready = 1;
                }
            }
            --ready;
            const uint8_t* pk = smem + st * C::kStage + C::kB;
#pragma unroll
            for (int gg = 0; gg < kIBK / KG; ++gg) {
                if (gg >= ngs) break;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                const int tile = 2 * warp + half;
                const uint32_t at = tmem + (uint32_t(16 * tile) << 16) + uint32_t(C::kACol0 + st * kIACols);
                const uint4 w = *reinterpret_cast<const uint4*>(pk + ((gg * kTilesPerBlock + tile) * 32 + lane) * 16);
                if (BITS == 4) {
                    // word j: row r0's codes of k-step j in the low nibbles, row r0 + 8's in the high
                    const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
                    uint32_t r[8];
#pragma unroll
                    for (int mm = 0; mm < 2; ++mm) {
                        const uint32_t w0 = wv[2 * mm], w1 = wv[2 * mm + 1];
                        r[4 * mm + 0] = nib4_to_s8(w0 & 0x0F0F0F0Fu);
                        r[4 * mm + 1] = nib4_to_s8(w1 & 0x0F0F0F0Fu);
                        r[4 * mm + 2] = nib4_to_s8((w0 >> 4) & 0x0F0F0F0Fu);
                        r[4 * mm + 3] = nib4_to_s8((w1 >> 4) & 0x0F0F0F0Fu);
                    }
                    tmem_st16x256_x2(at + uint32_t(16 * gg), r);  // 64 k: 16 columns
                } else {
                    // words 2j, 2j + 1: row r0's codes of k-step j in bytes 0-1 of
                    // each, row r0 + 8's in bytes 2-3; the stored code minus 128 is
                    // the code with its top bit flipped
                    uint32_t r[4];
                    r[0] = __byte_perm(w.x, w.y, 0x5410) ^ 0x80808080u;
                    r[1] = __byte_perm(w.z, w.w, 0x5410) ^ 0x80808080u;
                    r[2] = __byte_perm(w.x, w.y, 0x7632) ^ 0x80808080u;
                    r[3] = __byte_perm(w.z, w.w, 0x7632) ^ 0x80808080u;
                    tmem_st16x256_x1(at + uint32_t(8 * gg), r);  // 32 k: 8 columns
                }
                }
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&deq[st]));
            if (++st == STAGES) { st = 0; ph ^= 1u; }
        }
    } else if (warp >= kIFold0) {
        // ------------------------------------------------------- fold + epilogue
        // four warps per TMEM lane quarter; warp slice s takes the 16-column
        // chunks 16 s + 64 i of the token tile, row = the TMEM lane
        // four warps per TMEM lane quarter; warp slice s takes the 16 columns
        // 16 s .. 16 s + 15 of the token tile (tiles of at most 64), row = the
        // TMEM lane
        static_assert(BNMAX <= 64, "one 16-column chunk per fold warp");
        const int fw = warp - kIFold0;
        const int q = warp & 3, slice = fw >> 2;
        const int row = q * 32 + lane;
        const int tl = row >> 4, rr = row & 15;
        const int c0 = 16 * slice;
        const uint32_t lane_base = uint32_t(q * 32) << 16;
        // per-warp scratch: the 16 activation scales of the current block
        float* xsh = reinterpret_cast<float*>(bar_area + C::kScratchOff) + fw * 16;
        const bool short_blocks = a.block_size <= 256;
        int pb = 0;
        uint32_t pph = 0;
        int pready = 0;  // finished partials found ahead by the last batched test
        for (int i = blockIdx.x; i < total; i += gridDim.x) {
            const Item it = item_at(i, prefix, a, nrb, nks);
            const int ncol = ((it.rows + 15) / 16) * 16;
            const bool cols = c0 < ncol;  // uniform over the warp
            const int64_t p0 = it.seg0 + int64_t(it.tt) * a.bn;  // permuted row of column 0
            const int kb0 = k_lo(it) / a.block_size;
            const int nblk = (k_hi(it) - k_lo(it)) / a.block_size;
            // weight scale of this row, block 0 of the expert's 128-row block
            const int64_t sw0 = ((int64_t(it.e) * nrb + it.rb) * nsb) * (kTilesPerBlock * 16) + tl * 16 +
                                (rr & 7) * 2 + (rr >> 3);
            const int cj = c0 + (lane & 15);  // the column whose activation scale this lane fetches
            auto load_scales = [&](int bg, float& sw, float& xv) {
                const int64_t si = sw0 + int64_t(bg) * (kTilesPerBlock * 16);
                sw = a.scale_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(a.S)[si])
                                  : reinterpret_cast<const float*>(a.S)[si];
                xv = cj < it.rows ? a.xs[(p0 + cj) * nsb + bg] : 0.0f;
            };
            float acc[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) acc[j] = 0.0f;
            bool ok = true;
            float sw_n = 0.0f, xv_n = 0.0f;
            if (nblk > 0 && cols) load_scales(kb0, sw_n, xv_n);
            for (int b = 0; b < nblk; ++b) {
                // this block's scales were fetched during the previous block; the
                // next block's go out before the wait, so their latency hides
                const float sw = sw_n, xv = xv_n;
                if (b + 1 < nblk && cols) load_scales(kb0 + b + 1, sw_n, xv_n);
                if (pready == 0) {
                    pready = ready_run<C::kNPB - 1>(pfull, nullptr, pb, pph, 1, C::kNPB);
                    if (pready == 0) {
                        if (!warp_wait(smem_u32(&pfull[pb]), pph, abort_flag, a.status, a.timeout_ns)) { ok = false; break; }
                        pready = 1;
                    }
                }
                --pready;
                tc_fence_after();
                if (cols) {
                    // s_j = s_w * s_x of column c0 + j, through the warp's scratch
                    __syncwarp();
                    if (lane < 16) xsh[lane] = xv;
                    __syncwarp();
                    // two halves of 8 columns keep the live registers low
                    auto fold = [&](auto short_tag) {
                        constexpr bool SHORT = decltype(short_tag)::value;
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            uint32_t P[8];
                            tmem_ld8_u32(tmem + lane_base + uint32_t(pb * BNMAX + c0 + 8 * hh), P);
#pragma unroll
                            for (int j4 = 0; j4 < 2; ++j4) {
                                const float4 v = reinterpret_cast<const float4*>(xsh)[2 * hh + j4];
                                const float sv[4] = {sw * v.x, sw * v.y, sw * v.z, sw * v.w};
#pragma unroll
                                for (int e = 0; e < 4; ++e)
                                    acc[8 * hh + 4 * j4 + e] =
                                        fmaf(i32_to_f32_t<SHORT>(P[4 * j4 + e]), sv[e], acc[8 * hh + 4 * j4 + e]);
                            }
                        }
                    };
                    if (short_blocks)
                        fold(std::true_type{});
                    else
                        fold(std::false_type{});
                }
                if (b + 1 == nblk) break;  // the last partial's buffer stays held for the epilogue
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&pempty[pb]));
                if (++pb == C::kNPB) { pb = 0; pph ^= 1u; }
            }
            if (!ok) break;
            if (nblk > 0) {
                // the item's sum goes back into the last partial's columns (fp32)
                // for the shared epilogue, which reads them from there
                const uint32_t tb = tmem + lane_base + uint32_t(pb * BNMAX);
                if (cols) tmem_st16_f32(tb + uint32_t(c0), acc);
                tmem_st_wait();
                tc_epilogue_item<false>(a, it, nrb, tb, row, lane, c0, 64);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&pempty[pb]));
                if (++pb == C::kNPB) { pb = 0; pph ^= 1u; }
            }
            if (nblk == 0 && !a.is_fc1) {
                // an empty K range (more splits than stages): this split adds zero
                const int64_t prow = int64_t(it.rb) * kBlockRows + row;
                for (int c = c0; c < it.rows; c += 64)
                    for (int j = 0; j < 16 && c + j < it.rows; ++j)
                        if (prow < a.N)
                            reinterpret_cast<float*>(a.out)[(int64_t(it.split) * a.R + p0 + c + j) * a.N + prow] = 0.0f;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kIWarpMma) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
    }
}

// ---------------------------------------------------------------- host side

template <int BITS, int BNMAX>
struct LaunchI8 {
    static constexpr int kStage = I8Cfg<BITS, BNMAX, 1>::kStage;
    static constexpr int kByTmem = (512 - I8Cfg<BITS, BNMAX, 1>::kNPB * BNMAX) / kIACols;
    static constexpr int kBySmem = (200 * 1024) / kStage;
    static constexpr int kCap = kByTmem < kBySmem ? kByTmem : kBySmem;
    static constexpr int kStages = kCap < 12 ? kCap : 12;
    using C = I8Cfg<BITS, BNMAX, kStages>;
    static cudaError_t prepare() {
        return cudaFuncSetAttribute(ffn_tc_i8_kernel<BITS, BNMAX, kStages>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    C::kSmem);
    }
    static cudaError_t run(const CUtensorMap& map, const TcI8Args& a, int grid, cudaStream_t st) {
        ffn_tc_i8_kernel<BITS, BNMAX, kStages><<<grid, kIThreads, C::kSmem, st>>>(map, a);
        return cudaGetLastError();
    }
};

template <int BITS>
cudaError_t dispatch_i8(int bnmax, const CUtensorMap& map, const TcI8Args& a, int grid, cudaStream_t st) {
    switch (bnmax) {
        case 16: return LaunchI8<BITS, 16>::run(map, a, grid, st);
        case 32: return LaunchI8<BITS, 32>::run(map, a, grid, st);
        default: return LaunchI8<BITS, 64>::run(map, a, grid, st);
    }
}

template <int BITS>
cudaError_t prepare_i8_bits() {
    cudaError_t e = LaunchI8<BITS, 16>::prepare();
    if (e == cudaSuccess) e = LaunchI8<BITS, 32>::prepare();
    if (e == cudaSuccess) e = LaunchI8<BITS, 64>::prepare();
    return e;
}

}  // namespace

bool tc_i8_supports(int bits, int block_size, int64_t H, int64_t I) {
    (void)bits;
    // K blocks of 32 codes or more (one MMA is 32 k); K ranges split on
    // 128-k stages stay on block boundaries for blocks up to 128
    return block_size >= 32 && H % block_size == 0 && I % block_size == 0;
}

cudaError_t prepare_ffn_tc_i8() {
    cudaError_t e = prepare_i8_bits<4>();
    return e == cudaSuccess ? prepare_i8_bits<8>() : e;
}

cudaError_t launch_ffn_tc_i8(const FfnArgs& f, int bn, int32_t* status, cudaStream_t st) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    int bnmax = 16;
    while (bnmax < bn) bnmax *= 2;
    if (bnmax > 64 || f.block_size < 32 || !f.aq || !f.as) return cudaErrorInvalidConfiguration;
    // activation codes: [rows, K] bytes in the tensor-core order, rows = R
    CUtensorMap map;
    const cuuint64_t dims[2] = {cuuint64_t(f.K), cuuint64_t(f.R)};
    const cuuint64_t strides[1] = {cuuint64_t(f.K)};
    const cuuint32_t box[2] = {cuuint32_t(kIBK), cuuint32_t(bnmax < 64 ? bnmax : 64)};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t*>(f.aq), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    TcI8Args a{};
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
    a.xs = f.as;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return f.bits == 4 ? dispatch_i8<4>(bnmax, map, a, sms, st) : dispatch_i8<8>(bnmax, map, a, sms, st);
}

}  // namespace qmoe
