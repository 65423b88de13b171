// pack.cu -- one-time re-layout of the packed expert stacks into fragment
// order ("ClikaRT::nn::QMoEWoQ", initialize_impl(): the pack is the one
// resident copy; set_weights(): a re-bind drops the previous pack).
//
// Codes are moved, never decoded: the output has the input's byte count. The
// layout is described in qmoe_internal.cuh.
#include "qmoe_internal.cuh"

namespace qmoe {
namespace {

struct SrcRow {
    int which;   // 0 = src, 1 = src_up
    int64_t row; // row inside one expert of that source
};

// Source row of packed row rr of row tile rt.
__device__ __forceinline__ SrcRow source_row(int mode, int64_t rt, int rr, int64_t I) {
    if (mode == 0) return {0, rt * kTileRows + rr};
    const int64_t i = rt * 8 + (rr & 7);
    const int up = rr >= 8;
    if (mode == 1) return {0, 2 * i + up};      // fused, interleaved
    if (mode == 2) return {0, up ? I + i : i};  // fused, gate rows then up rows
    return {up, i};                             // gate from fc1, up from fc3
}

__device__ __forceinline__ int64_t source_rows(int mode, int64_t N, int64_t I) {
    return mode == 0 ? N : (mode == 3 ? I : 2 * I);
}

__device__ __forceinline__ uint32_t code_at(const uint8_t* rowp, int64_t k, int bits) {
    if (bits == 8) return rowp[k];
    const uint32_t b = rowp[k >> 1];
    return (k & 1) ? (b >> 4) : (b & 0xF);
}

// One thread writes the 16 bytes of one lane of one (row tile, k-group) unit.
// Units are ordered [E][N/128 row blocks][K/KG groups][8 row tiles]; row tiles
// past N (the padded tail of the last block) are written as zero codes.
__global__ void pack_codes_kernel(PackArgs a) {
    const int64_t nrt = a.N / kTileRows;
    const int64_t nrb = (nrt + kTilesPerBlock - 1) / kTilesPerBlock;
    const int kg = kgroup_of(a.bits);
    const int64_t ngr = a.K / kg;
    const int64_t total = a.E * nrb * ngr * kTilesPerBlock * 32;
    const int64_t src_rows = source_rows(a.mode, a.N, a.I);
    const int64_t row_bytes = a.K * a.bits / 8;
    for (int64_t id = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; id < total;
         id += (int64_t)gridDim.x * blockDim.x) {
        const int lane = int(id & 31);
        int64_t rest = id >> 5;
        const int64_t tib = rest % kTilesPerBlock;
        rest /= kTilesPerBlock;
        const int64_t g = rest % ngr;
        rest /= ngr;
        const int64_t rb = rest % nrb;
        const int64_t e = rest / nrb;
        const int64_t rt = rb * kTilesPerBlock + tib;
        const int r0 = lane >> 2, c = lane & 3;
        uint32_t words[4] = {0u, 0u, 0u, 0u};
        if (rt < nrt && a.bits == 4) {
            // word j, nibble p: row r0 + 8*(p&1), k = 64g + 16j + 4c + 2*((p>>1)&1) + (p>>2)
            for (int j = 0; j < 4; ++j) {
                uint32_t w = 0;
                for (int p = 0; p < 8; ++p) {
                    const int rr = r0 + 8 * (p & 1);
                    const int64_t k = g * 64 + 16 * j + 4 * c + 2 * ((p >> 1) & 1) + (p >> 2);
                    const SrcRow s = source_row(a.mode, rt, rr, a.I);
                    const uint8_t* base = s.which ? a.src_up : a.src;
                    const uint8_t* rowp = base + (e * src_rows + s.row) * row_bytes;
                    w |= code_at(rowp, k, 4) << (4 * p);
                }
                words[j] = w;
            }
        } else if (rt < nrt) {
            // kstep j (8 bytes), byte m: pair q = m/2 -> row r0 + 8*(q&1),
            // k = 32g + 16j + 4c + 2*(q>>1) + (m&1)
            for (int j = 0; j < 2; ++j) {
                for (int half = 0; half < 2; ++half) {
                    uint32_t w = 0;
                    for (int mb = 0; mb < 4; ++mb) {
                        const int m = half * 4 + mb;
                        const int q = m >> 1;
                        const int rr = r0 + 8 * (q & 1);
                        const int64_t k = g * 32 + 16 * j + 4 * c + 2 * (q >> 1) + (m & 1);
                        const SrcRow s = source_row(a.mode, rt, rr, a.I);
                        const uint8_t* base = s.which ? a.src_up : a.src;
                        const uint8_t* rowp = base + (e * src_rows + s.row) * row_bytes;
                        w |= code_at(rowp, k, 8) << (8 * mb);
                    }
                    words[2 * j + half] = w;
                }
            }
        }
        uint4 v = make_uint4(words[0], words[1], words[2], words[3]);
        *reinterpret_cast<uint4*>(a.dst + id * 16) = v;
    }
}

// Scales: [E][N/128 row blocks][K/bs or 1][8 row tiles][16], the 16 entries
// of a row tile in lane order (r0, r0 + 8) pairs; padded tiles hold zeros.
__global__ void pack_scales_kernel(PackArgs a) {
    const int64_t nrt = a.N / kTileRows;
    const int64_t nrb = (nrt + kTilesPerBlock - 1) / kTilesPerBlock;
    const int64_t nsb = a.block_size > 0 ? a.K / a.block_size : 1;
    const int64_t total = a.E * nrb * nsb * kTilesPerBlock * 16;
    const int64_t src_rows = source_rows(a.mode, a.N, a.I);
    for (int64_t id = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; id < total;
         id += (int64_t)gridDim.x * blockDim.x) {
        const int pos = int(id & 15);
        int64_t rest = id >> 4;
        const int64_t tib = rest % kTilesPerBlock;
        rest /= kTilesPerBlock;
        const int64_t b = rest % nsb;
        rest /= nsb;
        const int64_t rb = rest % nrb;
        const int64_t e = rest / nrb;
        const int64_t rt = rb * kTilesPerBlock + tib;
        const int rr = (pos >> 1) + 8 * (pos & 1);
        if (rt >= nrt) {
            if (a.scale_bf16)
                ((uint16_t*)a.s_dst)[id] = 0;
            else
                ((float*)a.s_dst)[id] = 0.0f;
            continue;
        }
        const SrcRow s = source_row(a.mode, rt, rr, a.I);
        const int64_t src_idx = (e * src_rows + s.row) * nsb + b;
        if (a.scale_e8m0) {
            // E8M0 byte x is 2^(x - 127): the bf16 with exponent field x and an
            // empty mantissa, bit for bit (x = 0 gives 2^-127 as a subnormal)
            const uint8_t x = ((const uint8_t*)(s.which ? a.s_src_up : a.s_src))[src_idx];
            ((uint16_t*)a.s_dst)[id] = x == 0 ? uint16_t(0x0040) : uint16_t(uint16_t(x) << 7);
        } else if (a.scale_bf16) {
            const uint16_t* src = (const uint16_t*)(s.which ? a.s_src_up : a.s_src);
            ((uint16_t*)a.s_dst)[id] = src[src_idx];
        } else {
            const float* src = (const float*)(s.which ? a.s_src_up : a.s_src);
            ((float*)a.s_dst)[id] = src[src_idx];
        }
    }
}

__device__ __forceinline__ float load_act(const void* p, int64_t i, int bf16) {
    if (bf16) return __bfloat162float(((const __nv_bfloat16*)p)[i]);
    return ((const float*)p)[i];
}

__global__ void pack_bias_kernel(PackArgs a) {
    const int64_t total = a.E * a.N;
    const int64_t src_rows = source_rows(a.mode, a.N, a.I);
    for (int64_t id = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; id < total;
         id += (int64_t)gridDim.x * blockDim.x) {
        const int64_t n = id % a.N, e = id / a.N;
        const SrcRow s = source_row(a.mode, n / kTileRows, int(n % kTileRows), a.I);
        const void* src = s.which ? a.b_src_up : a.b_src;
        a.b_dst[id] = src ? load_act(src, e * src_rows + s.row, a.act_bf16) : 0.0f;
    }
}

int grid_for(int64_t n, int threads) {
    int64_t b = (n + threads - 1) / threads;
    if (b > 148 * 64) b = 148 * 64;
    return int(b < 1 ? 1 : b);
}

}  // namespace

cudaError_t launch_pack(const PackArgs& a, cudaStream_t st) {
    const int th = 256;
    const int64_t nrb = padded_rows(a.N) / kBlockRows;
    const int64_t ncode = a.E * nrb * (a.K / kgroup_of(a.bits)) * kTilesPerBlock * 32;
    pack_codes_kernel<<<grid_for(ncode, th), th, 0, st>>>(a);
    const int64_t nsb = a.block_size > 0 ? a.K / a.block_size : 1;
    pack_scales_kernel<<<grid_for(a.E * nrb * nsb * kTilesPerBlock * 16, th), th, 0, st>>>(a);
    if (a.b_dst) pack_bias_kernel<<<grid_for(a.E * a.N, th), th, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace qmoe
