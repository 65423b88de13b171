// ffn_tc_wide.cu -- expert FFN layers on the tcgen05 tensor cores for wide
// token tiles (up to 256 routed rows of one expert per tile), sm_100a.
//
// Same contraction as ffn_tc.cu -- y = x @ dequant(W).T + b per expert
// ("QLinearWoQ" page, class summary), the packed weights decoded one 128 x 64
// tile at a time inside the loop ("ClikaRT::nn::QMoEWoQ", class description)
// -- for experts with many routed rows. Decoding costs the same per weight
// whatever the token count, so a wider token tile (N = 256 in one
// 128 x 256 x 16 MMA) halves the decode work per FLOP against N = 128. Two
// N = 256 fp32 accumulators fill all 512 TMEM columns, so here the decoded A
// tile goes to shared memory (128-byte swizzled K-major rows, the layout the
// MMA's shared-memory descriptor reads) instead of TMEM, and the MMA takes
// both operands from shared memory.
//
// Warp roles (864 threads, one CTA per SM):
//   warps 0-15  dequantise: two groups of eight take alternate stages; a warp
//               decodes one 16-row tile into a ring of shared-memory A slots
//               (st.shared, then an async-proxy fence)
//   warp 16     activation producer: 64-row TMA boxes (up to four per stage)
//   warp 26     weight producer: packed 128 x 64 tile and its scales (bulk)
//   warp 17     TMEM allocation and MMA issue (converged warp, elected lane)
//   warps 18-25 epilogue, shared with ffn_tc.cu
// Every wait is bounded (about two seconds, then QMOE_TIMEOUT in the
// workspace status word; every role leaves its loop and the CTA frees TMEM).
#include "qmoe_internal.cuh"
#include "tc_common.cuh"
#include "fp4_decode.cuh"

namespace qmoe {
namespace {

constexpr int kWBK = 64;             // k per stage
constexpr int kWN = 256;             // token-tile width (MMA N)
constexpr int kWDeqWarps = 16;            // two groups of 8, alternate stages
constexpr int kWWarpProd = 16;
constexpr int kWWarpMma = 17;
constexpr int kWEpi0 = 18;
constexpr int kWEpiWarps = 8;
constexpr int kWWarpProd2 = kWEpi0 + kWEpiWarps;  // 26
constexpr int kWThreads = (kWWarpProd2 + 1) * 32;  // 864
constexpr int kWScaleMax = 4 * kTilesPerBlock * 16 * 4;  // four blocks of fp32 pairs

template <int BITS>
struct WideCfg {
    static constexpr int kBoxRows = 64;
    static constexpr int kB = kWN * 128;                       // activation tile, 32 KB
    static constexpr int kPacked = kBlockRows * kWBK * BITS / 8;
    static constexpr int kStage = kB + kPacked + kWScaleMax;   // activations, codes, scales
    static constexpr int kA = kBlockRows * 128;                // decoded A tile, 16 KB
    static constexpr int kAS = BITS == 4 ? 4 : 3;              // A-tile slots
    static constexpr int kStages = (222 * 1024 - kAS * kA) / kStage;  // 4 (int4) / 4 (int8)
    static constexpr int kAOff = kStages * kStage;             // multiple of 1024
    static constexpr int kBarOff = kAOff + kAS * kA;
    static constexpr int kBarBytes = 2048;
    static constexpr int kPrefixOff = 512;
    static constexpr int kSmem = kBarOff + kBarBytes + 1024;
    static_assert(kStage % 1024 == 0 && kA % 1024 == 0, "1024-byte aligned slots");
    static_assert(kStages >= 3 && kSmem <= 227 * 1024, "shared-memory budget");
};

template <int BITS, bool PERCOL, bool FP4>
__global__ void __launch_bounds__(kWThreads, 1)
    ffn_tc_wide_kernel(const __grid_constant__ CUtensorMap bmap, const TcArgs a) {
    using C = WideCfg<BITS>;
    constexpr int ST = C::kStages, AS = C::kAS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint8_t* asm_ = smem + C::kAOff;                  // decoded A tiles
    uint8_t* bar_area = smem + C::kBarOff;
    uint64_t* full = reinterpret_cast<uint64_t*>(bar_area);  // stage landed (both producers)
    uint64_t* empty = full + ST;                              // stage read by the MMAs
    uint64_t* afull = empty + ST;                             // A tile written
    uint64_t* aempty = afull + AS;                            // A tile read by the MMAs
    uint64_t* accf = aempty + AS;
    uint64_t* acce = accf + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acce + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* prefix = reinterpret_cast<int*>(bar_area + C::kPrefixOff);

    const int nrb = int(padded_rows(a.N) / kBlockRows);
    const int nks = int(a.K / kWBK);

    if (tid == 0) {
        for (int s = 0; s < ST; ++s) {
            mbar_init(smem_u32(&full[s]), 2);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        for (int s = 0; s < AS; ++s) {
            mbar_init(smem_u32(&afull[s]), kWDeqWarps / 2);  // one group writes a slot
            mbar_init(smem_u32(&aempty[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&accf[b]), 1);
            mbar_init(smem_u32(&acce[b]), kWEpiWarps);
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
    if (warp == kWWarpMma) {
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
    const int nsb = a.block_size > 0 ? int(a.K / a.block_size) : 1;
    const int ssz = a.scale_bf16 ? 2 : 4;
    const int sblk = PERCOL ? 0 : (a.block_size >= kWBK ? 1 : kWBK / a.block_size);
    const uint32_t sbytes = uint32_t(sblk * kTilesPerBlock * 16 * ssz);

    if (warp == kWWarpProd || warp == kWWarpProd2) {
        // ------------------------------------------------------- producers
        const bool acts = warp == kWWarpProd;
        const uint32_t e = elect_one();
        int st = 0;
        uint32_t ph = 0;
        bool ok = true;
        const int ngr = int(a.K / kgroup_of(BITS));
        const int bs_log2 = PERCOL ? 0 : __ffs(a.block_size) - 1;
        for (int i = blockIdx.x; ok && i < total; i += gridDim.x) {
            const Item it = item_at(i, prefix, a, nrb, nks);
            const int nbox = (it.rows + C::kBoxRows - 1) / C::kBoxRows;
            const uint32_t bytes = acts ? uint32_t(nbox * C::kBoxRows * 128) : uint32_t(C::kPacked) + sbytes;
            const int y0 = int(it.seg0) + it.tt * a.bn;
            const int64_t blk = int64_t(it.e) * nrb + it.rb;
            for (int ks = it.ks_lo; ks < it.ks_hi; ++ks) {
                if (!warp_wait(smem_u32(&empty[st]), ph ^ 1u, abort_flag, a.status, a.timeout_ns)) { ok = false; break; }
                uint8_t* sb = smem + st * C::kStage;
                const uint32_t fb = smem_u32(&full[st]);
                mbar_expect_tx_e(fb, bytes, e);
                if (acts) {
                    for (int b = 0; b < nbox; ++b)
                        tma_2d_e(smem_u32(sb + b * C::kBoxRows * 128), &bmap, ks * kWBK, y0 + b * C::kBoxRows, fb, e);
                } else {
                    const int g = ks * (kWBK / kgroup_of(BITS));
                    const uint8_t* src = a.W + (blk * ngr + g) * int64_t(kTilesPerBlock) * kUnitBytes;
                    bulk_g2s_e(smem_u32(sb + C::kB), src, C::kPacked, fb, e);
                    if (!PERCOL) {
                        const int b0 = (ks * kWBK) >> bs_log2;
                        const uint8_t* ssrc = reinterpret_cast<const uint8_t*>(a.S) +
                                              (blk * nsb + b0) * int64_t(kTilesPerBlock * 16 * ssz);
                        bulk_g2s_e(smem_u32(sb + C::kB + C::kPacked), ssrc, sbytes, fb, e);
                    }
                }
                if (++st == ST) { st = 0; ph ^= 1u; }
            }
        }
    } else if (warp == kWWarpMma) {
        // ------------------------------------------------------- MMA issue
        const uint32_t e = elect_one();
        int st = 0, as = 0, acc = 0;
        uint32_t ph = 0, aph = 0, cph = 0;
        bool ok = true;
        for (int i = blockIdx.x; ok && i < total; i += gridDim.x) {
            const Item it = item_at(i, prefix, a, nrb, nks);
            const uint32_t idesc = idesc_bf16(((it.rows + 15) / 16) * 16);
            if (!warp_wait(smem_u32(&acce[acc]), cph ^ 1u, abort_flag, a.status, a.timeout_ns)) break;
            tc_fence_after();
            const uint32_t d = tmem + uint32_t(acc * kWN);
            for (int ks = it.ks_lo; ks < it.ks_hi; ++ks) {
                if (!warp_wait(smem_u32(&full[st]), ph, abort_flag, a.status, a.timeout_ns) ||
                    !warp_wait(smem_u32(&afull[as]), aph, abort_flag, a.status, a.timeout_ns)) { ok = false; break; }
                tc_fence_after();
                const uint64_t ad = desc_sw128(smem_u32(asm_ + as * C::kA));
                const uint64_t bd = desc_sw128(smem_u32(smem + st * C::kStage));
                const uint32_t acc0 = ks > it.ks_lo ? 1u : 0u;
#pragma unroll
                for (int kk = 0; kk < kWBK / 16; ++kk)  // 16 k per MMA: 32 B into each swizzled row
                    mma_bf16_ss_e(d, ad + uint64_t(2 * kk), bd + uint64_t(2 * kk), idesc, kk > 0 ? 1u : acc0, e);
                mma_commit_e(smem_u32(&empty[st]), e);
                mma_commit_e(smem_u32(&aempty[as]), e);
                if (++st == ST) { st = 0; ph ^= 1u; }
                if (++as == AS) { as = 0; aph ^= 1u; }
            }
            if (!ok) break;
            // test hook: with a.withhold the first item's accumulator is never
            // announced, so the epilogue's bounded wait runs out (no fault)
            mma_commit_e(smem_u32(&accf[acc]), (a.withhold && i == int(blockIdx.x)) ? 0u : e);
            if (++acc == 2) { acc = 0; cph ^= 1u; }
        }
    } else if (warp < kWDeqWarps) {
        // ------------------------------------------------------- dequantise
        // warp w decodes row tile w % 8 (rows 16 (w % 8) .. + 15 of the 128-row
        // block) of the stages of parity w / 8: two groups of eight warps take
        // alternate stages, so two stages are decoded at once
        const int tile = warp & 7, grp = warp >> 3;
        int seen = 0;  // stages seen by this warp, both parities
        const int r0 = lane >> 2, c = lane & 3;
        const int rA = 16 * tile + r0;  // and rA + 8; both have (row & 7) == r0
        int st = 0, as = 0;
        uint32_t ph = 0, aph = 0;
        bool ok = true;
        const uint32_t kMask = 0x000F000Fu, kMagic = 0x43004300u, kBias4 = 0x43084308u;
        const int bs_shift = a.block_size >= kWBK ? 30 : __ffs(a.block_size) - 1;
        for (int i = blockIdx.x; ok && i < total; i += gridDim.x) {
            const Item it = item_at(i, prefix, a, nrb, nks);
            for (int ks = it.ks_lo; ks < it.ks_hi; ++ks) {
                if ((seen++ & 1) != grp) {  // the other group's stage
                    if (++st == ST) { st = 0; ph ^= 1u; }
                    if (++as == AS) { as = 0; aph ^= 1u; }
                    continue;
                }
                if (!warp_wait(smem_u32(&full[st]), ph, abort_flag, a.status, a.timeout_ns) ||
                    !warp_wait(smem_u32(&aempty[as]), aph ^ 1u, abort_flag, a.status, a.timeout_ns)) { ok = false; break; }
                const uint8_t* pk = smem + st * C::kStage + C::kB;
                const uint8_t* sc = pk + C::kPacked;
                uint8_t* at = asm_ + as * C::kA;
                constexpr int GROUPS = kWBK / kgroup_of(BITS);  // 1 (int4) or 2 (int8)
                constexpr int KSTEPS = kgroup_of(BITS) / 16;
#pragma unroll
                for (int gg = 0; gg < GROUPS; ++gg) {
                    const uint4 w = *reinterpret_cast<const uint4*>(pk + ((gg * kTilesPerBlock + tile) * 32 + lane) * 16);
                    const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
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
#pragma unroll
                            for (int qq = 0; qq < 4; ++qq) {
                                const uint32_t word = wv[2 * j + (qq >> 1)];
                                const uint32_t pr = __byte_perm(word, 0u, (qq & 1) ? 0x4342u : 0x4140u);
                                const uint32_t lo = (pr & 0x007F007Fu) | 0x43004300u;
                                const uint32_t hi = (pr & 0x00800080u) ^ 0x43804380u;
                                A[qq] = bf2_sub(lo, hi);
                            }
                        }
                        const int ks16 = gg * KSTEPS + j;  // 16-k step inside the 64-k stage
                        if (!PERCOL) {
                            const int kl = 16 * ks16 + 4 * c;
                            const int si = ((kl >> bs_shift) * kTilesPerBlock + tile) * 16 + 2 * r0;
                            uint32_t sa2, sb2;
                            if (a.scale_bf16) {
                                const uint32_t raw = *reinterpret_cast<const uint32_t*>(sc + si * 2);
                                sa2 = __byte_perm(raw, 0u, 0x1010);
                                sb2 = __byte_perm(raw, 0u, 0x3232);
                            } else {
                                const float2 f = *reinterpret_cast<const float2*>(sc + si * 4);
                                sa2 = bf2_bcast(f.x);
                                sb2 = bf2_bcast(f.y);
                            }
                            A[0] = bf2_mul(A[0], sa2);
                            A[2] = bf2_mul(A[2], sa2);
                            A[1] = bf2_mul(A[1], sb2);
                            A[3] = bf2_mul(A[3], sb2);
                        }
                        // k = 16*ks16 + 4c .. +3 of rows rA and rA + 8: 8 bytes at byte
                        // 32*ks16 + 8c of each 128-byte row; 16-byte chunk index XOR
                        // (row & 7) is the 128-byte swizzle
                        const int chunk = (2 * ks16 + (c >> 1)) ^ r0;
                        const int off = chunk * 16 + 8 * (c & 1);
                        *reinterpret_cast<uint2*>(at + rA * 128 + off) = make_uint2(A[0], A[2]);
                        *reinterpret_cast<uint2*>(at + (rA + 8) * 128 + off) = make_uint2(A[1], A[3]);
                    }
                }
                // generic-proxy stores -> visible to the tensor core's async proxy
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&afull[as]));
                if (++st == ST) { st = 0; ph ^= 1u; }
                if (++as == AS) { as = 0; aph ^= 1u; }
            }
        }
    } else if (warp >= kWEpi0 && warp < kWEpi0 + kWEpiWarps) {
        // ------------------------------------------------------- epilogue
        const int qd = warp & 3;                   // TMEM lane quarter this warp may read
        const int half = (warp - kWEpi0) >> 2;     // which 16-column chunks it takes
        const int row = qd * 32 + lane;
        int acc = 0;
        uint32_t cph = 0;
        for (int i = blockIdx.x; i < total; i += gridDim.x) {
            const Item it = item_at(i, prefix, a, nrb, nks);
            if (!warp_wait(smem_u32(&accf[acc]), cph, abort_flag, a.status, a.timeout_ns)) break;
            tc_fence_after();
            tc_epilogue_item<PERCOL>(a, it, nrb, tmem + (uint32_t(qd * 32) << 16) + uint32_t(acc * kWN), row, lane,
                                     16 * half, 32);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&acce[acc]));
            if (++acc == 2) { acc = 0; cph ^= 1u; }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kWWarpMma) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
    }
}

template <int BITS, bool PERCOL, bool FP4>
cudaError_t prepare_one() {
    return cudaFuncSetAttribute(ffn_tc_wide_kernel<BITS, PERCOL, FP4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                WideCfg<BITS>::kSmem);
}

}  // namespace

cudaError_t prepare_ffn_tc_wide() {
    cudaError_t e = prepare_one<4, false, false>();
    if (e == cudaSuccess) e = prepare_one<4, true, false>();
    if (e == cudaSuccess) e = prepare_one<8, false, false>();
    if (e == cudaSuccess) e = prepare_one<8, true, false>();
    if (e == cudaSuccess) e = prepare_one<4, false, true>();  // MXFP4
    return e;
}

cudaError_t launch_ffn_tc_wide(const FfnArgs& f, int bn, int32_t* status, cudaStream_t st) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    if (bn > kWN || bn < 1 || f.E + 1 > (2048 - 512) / 4) return cudaErrorInvalidValue;
    CUtensorMap map;
    const cuuint64_t dims[2] = {cuuint64_t(f.K), cuuint64_t(f.R)};
    const cuuint64_t strides[1] = {cuuint64_t(f.K * 2)};
    const cuuint32_t box[2] = {cuuint32_t(kWBK), 64u};
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
    void (*kern)(const CUtensorMap, const TcArgs) =
        f.bits == 4 ? (f.fp4    ? ffn_tc_wide_kernel<4, false, true>
                       : percol ? ffn_tc_wide_kernel<4, true, false>
                                : ffn_tc_wide_kernel<4, false, false>)
                    : (percol ? ffn_tc_wide_kernel<8, true, false> : ffn_tc_wide_kernel<8, false, false>);
    const int smem = f.bits == 4 ? WideCfg<4>::kSmem : WideCfg<8>::kSmem;
    kern<<<sms, kWThreads, smem, st>>>(map, a);
    return cudaGetLastError();
}

}  // namespace qmoe
