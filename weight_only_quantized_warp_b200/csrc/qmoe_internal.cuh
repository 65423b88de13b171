// qmoe_internal.cuh -- declarations shared by the CUDA translation units of
// the QMoE library: the handle, the per-call plan, the packed weight layout
// and the kernel launchers. Nothing here is part of the public C ABI.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <string>
#include <utility>

#include "qmoe.h"

namespace qmoe {

// ---------------------------------------------------------------------------
// Programmatic dependent launch. A kernel launched with pdl = true may start
// while the kernel before it on the stream is still running; it must call
// pdl_wait() before it reads anything that kernel (or an earlier one) wrote.
// pdl_trigger() lets the next kernel's launch begin once every CTA of this
// grid has called it or exited. Both are no-ops when no such launch is
// involved.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                 bool pdl, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// ---------------------------------------------------------------------------
// Packed weight layout ("fragment order").
//
// A weight W[N, K] of one expert (N output rows, K reduction) is cut into row
// tiles of 16 rows and k-groups of KG (64 for 4-bit codes, 32 for 8-bit). One
// (row tile, k-group) unit is 512 bytes: lane L of a warp owns rows r0 = L/4
// and r0 + 8 of the tile and, with c = L%4, the k values 16j + 4c + {0..3}
// of the group for j = 0 .. KG/16 - 1 -- 16 bytes. Word (int4) or word pair
// (int8) j holds the codes of k-step j in the order of the m16n8k16 MMA A
// fragment, which is also the register order of a 16x256b tensor-memory
// store: registers (row r0, k 16j+4c+{0,1}), (row r0+8, same), (row r0,
// k 16j+4c+{2,3}), (row r0+8, same). Units are ordered [N/128 row blocks]
// [K/KG groups][8 row tiles], so a 128-row x KG slab (one tensor-core stage)
// is one contiguous 4 KB run and a row tile walks K with a 4 KB stride. N is
// padded to a multiple of 128 with zero codes. Bytes are the page's codes,
// re-laid, never decoded.
//
// FC1 of a gated FFN is re-laid so that row tile t holds gate rows
// i = 8t..8t+7 in its first 8 rows and the matching up rows in its last 8,
// whatever the input layout (fused interleaved, fused concatenated, or fc1 +
// fc3). Scales follow as [N/128][K/bs or 1][8 row tiles][16] with the 16
// entries of a tile in lane order (r0, r0 + 8) pairs; biases as fp32 in
// packed row order.
// ---------------------------------------------------------------------------
constexpr int kTileRows = 16;
constexpr int kTilesPerBlock = 8;
constexpr int kBlockRows = kTileRows * kTilesPerBlock;  // 128
constexpr int kUnitBytes = 512;
__host__ __device__ constexpr int kgroup_of(int bits) { return bits == 4 ? 64 : 32; }
__host__ __device__ constexpr int64_t padded_rows(int64_t n) {
    return (n + kBlockRows - 1) / kBlockRows * kBlockRows;
}

// Activation code passed to the kernels for GELU in its tanh form
// (activation_type GELU with gelu_mode QMOE_GELU_TANH); the other codes are
// the public QMOE_ACT_* values.
constexpr int kActGeluTanh = 5;

// Hot-path selection.
enum Path : int { kPathSimt = 0, kPathDecode = 1, kPathTc = 2, kPathTcDecode = 3, kPathI8 = 4, kPathI8Tc = 5 };

struct Plan {
    int path = kPathDecode;
    int64_t T = 0, R = 0;
    int nt = 1;          // 8-token MMA n-tiles handled per pass (decode path)
    int fc2_splits = 1;  // split-K factor of FC2 (partials reduced by the combine)
    int launches = 0;
    bool ok = true;      // a kernel configuration exists for this shape
    int bn = 0;          // token tile of the tensor-core path
    bool fused_route = false;  // routing and permutation in one launch (few tokens)
    bool gather = false;       // routed rows of x gathered (and weighted) into the workspace
    size_t off_idx = 0, off_w = 0, off_inv = 0, off_perm = 0, off_offsets = 0, off_status = 0,
           off_h = 0, off_o = 0, off_xperm = 0, total = 0;
    // int8 block tier: codes and block scales of FC1's input rows (x, or the
    // gathered rows) and of h
    int64_t xq_rows = 0;
    size_t off_xq = 0, off_xs = 0, off_hq = 0, off_hs = 0;
};

}  // namespace qmoe

struct qmoe_handle {
    qmoe_config cfg{};
    bool gated = false;
    int64_t n1 = 0;       // packed FC1 rows: 2I gated, I otherwise
    bool bound = false;
    uint8_t* w1 = nullptr;
    void* s1 = nullptr;
    float* b1 = nullptr;  // packed-row-order fp32, nullptr when no fc1/fc3 bias
    uint8_t* w2 = nullptr;
    void* s2 = nullptr;
    float* b2 = nullptr;  // [E, H] fp32, nullptr when no fc2 bias
    int device = -1;
    int path_override = -1;  // QMOE_OPT_PATH; -1 = choose by shape
    int decode_tiles = 0;    // QMOE_OPT_DECODE_TILES; 0 = choose by shape
    float* score_bias = nullptr;  // e_score_correction_bias [E] fp32, or nullptr
    uint64_t wait_limit_ns = 2000000000ull;  // QMOE_OPT_WAIT_LIMIT_NS
    int withhold = 0;        // QMOE_OPT_TEST_WITHHOLD
    int pdl = 1;             // QMOE_OPT_PDL
    mutable std::mutex mu;
    mutable std::string last_error;
};

namespace qmoe {

// rows_mode: T pre-routed rows, one expert each (the expert-parallel rows
// entry): R = T, and no router-weighted gather.
Plan make_plan(const qmoe_handle& h, int64_t T, bool rows_mode = false);

// ----------------------------------------------------------------- launchers
// Each returns the cudaError_t of its launch.

// Re-lay one packed stack (and its scales / biases) into fragment order.
// Row mapping: mode 0 = identity; 1 = fused interleaved gate/up; 2 = fused
// concatenated gate/up; 3 = gate from `src`, up from `src_up` (fc1 + fc3).
struct PackArgs {
    const uint8_t* src;
    const uint8_t* src_up;   // mode 3 only
    const void* s_src;
    const void* s_src_up;    // mode 3 only
    const void* b_src;       // nullable
    const void* b_src_up;    // nullable (mode 3)
    uint8_t* dst;
    void* s_dst;
    float* b_dst;            // nullable
    int64_t E, N, K;         // N = packed rows of one expert
    int64_t I;               // gated modes: inter size
    int bits, block_size, mode;
    int scale_bf16, act_bf16;
    int scale_e8m0;          // source scales are E8M0 bytes, packed as bf16
};
cudaError_t launch_pack(const PackArgs& a, cudaStream_t st);

// Top-k softmax routing: warp per token. sbias (nullable): per-expert bias of
// the selection keys.
cudaError_t launch_route(const void* logits, int act_bf16, int64_t T, int E, int k, int normalize, int n_group,
                         int topk_group, const float* sbias, int32_t* topk_idx, float* topk_w, int32_t* status,
                         cudaStream_t st);
// Routing and permutation of at most kFusedRouteTokens tokens in one launch.
constexpr int64_t kFusedRouteTokens = 64;
cudaError_t launch_route_permute(const void* logits, int act_bf16, int64_t T, int E, int k, int normalize,
                                 int n_group, int topk_group, const float* sbias, int32_t* topk_idx, float* topk_w,
                                 int32_t* offsets, int32_t* perm_tok, int32_t* inv, int32_t* status,
                                 cudaStream_t st);

// Histogram, scan and stable scatter into per-expert segments (one CTA).
// prepare_route_permute() raises the permute kernel's shared-memory limit on
// the current device; call it once per device before the first launch.
cudaError_t prepare_route_permute();
cudaError_t launch_permute(const int32_t* topk_idx, int64_t T, int E, int k, int32_t* offsets,
                           int32_t* perm_tok, int32_t* inv, cudaStream_t st);
// Expert parallel: the expert of every segment-ordered row
// (row_expert[inv[s]] = topk_idx[s]), and caller-given global expert ids
// rebased to a handle's local ids (id - base); an id outside [0, E) becomes
// expert 0 and sets QMOE_INVALID_ARGUMENT in the status word, so no later
// kernel indexes out of range.
cudaError_t launch_scatter_row_experts(const int32_t* topk_idx, const int32_t* inv, int64_t R, int32_t* row_expert,
                                       cudaStream_t st);
cudaError_t launch_rebase_experts(const int32_t* ids, int64_t R, int32_t base, int E, int32_t* local,
                                  int32_t* status, cudaStream_t st);

// Expert FFN layer over the segments (decode / SIMT paths).
struct FfnArgs {
    const uint8_t* W;        // packed weights, fragment order
    const void* S;           // packed scales
    const float* bias;       // packed-row-order fp32 (FC1), or nullptr
    const void* act;         // activations: x [T, K] (FC1) or h [R, K] (FC2)
    const int32_t* rowmap;   // perm_tok for FC1 (row of x), nullptr for FC2
    const int32_t* offsets;  // [E + 1]
    void* out;               // FC1: h [R, I]; FC2: partials [splits, R, N] fp32
    int64_t N, K, R;
    int E, bits, block_size;
    int gated, is_fc1, act_type;
    float alpha, beta, limit;
    int splits;
    int scale_bf16, act_bf16;
    int nt;
    int fp4;                 // codes are MXFP4 e2m1 (no zero point)
    // int8 block tier: the activation rows as codes [rows, K] (for 4-bit
    // weights every run of 4 codes in the order k+0, k+2, k+1, k+3) and
    // per-block scales [rows, K / block_size]; rows indexed like `act`
    const int8_t* aq;
    const float* as;
    // tcgen05 kernels: limit of every bounded device wait, and the test-only
    // withheld accumulator signal (QMOE_OPT_WAIT_LIMIT_NS, QMOE_OPT_TEST_WITHHOLD)
    uint64_t timeout_ns;
    int withhold;
    // weight-streaming decode kernel: launched as a programmatic dependent of
    // the kernel before it (prefetches weights, then waits for its inputs)
    int pdl;
};
cudaError_t launch_ffn_decode(const FfnArgs& a, cudaStream_t st);
// Shared memory of one decode CTA (staged activation rows) and its limit;
// prepare_ffn_decode() raises the kernels' limit on the current device.
constexpr size_t kDecodeSmemLimit = 200 * 1024;
constexpr int64_t kDecodeSmemTarget = 112 * 1024;  // at least two CTAs per SM (three fit below 75 KB)
// Rows per expert up to which the weight-streaming kernels are chosen (one
// 8-token tile per pass; above it the tensor-core GEMM decodes each weight
// once per token tile of up to 256 rows, measured faster from 16 rows per
// expert on).
constexpr int64_t kDecodeRowsPerExpert = 8;
int64_t decode_smem_bytes(int64_t K, int bits, int block_size, int splits, int nt);
cudaError_t prepare_ffn_decode();
cudaError_t launch_ffn_simt(const FfnArgs& a, cudaStream_t st);

// The int8 block tier on the tensor cores (tcgen05 kind::i8): activation
// codes [R, K] in the tensor-core order of quantize layouts 2 / 3 (f.aq),
// their block scales [R, K / block_size] (f.as), token tile bn <= 64.
// tc_i8_supports: the shapes it takes (blocks of at least 32 codes).
bool tc_i8_supports(int bits, int block_size, int64_t H, int64_t I);
cudaError_t prepare_ffn_tc_i8();
cudaError_t launch_ffn_tc_i8(const FfnArgs& f, int bn, int32_t* status, cudaStream_t st);

// Tensor-core (tcgen05) expert FFN layer over the segments; bn = token tile.
// prepare_ffn_tc() raises the kernels' shared-memory limit on the current
// device. launch_gather_rows copies the routed rows of x into segment order.
cudaError_t prepare_ffn_tc();
cudaError_t launch_ffn_tc(const FfnArgs& a, int bn, int32_t* status, cudaStream_t st);
// Token tiles wider than 128 (up to 256): A tile in shared memory, N = 256 MMAs.
cudaError_t prepare_ffn_tc_wide();
cudaError_t launch_ffn_tc_wide(const FfnArgs& a, int bn, int32_t* status, cudaStream_t st);
// Tensor-core streaming decode (few rows per expert; activations resident in
// shared memory): tc_decode_fits says whether a K range split `splits` ways
// fits its resident-activation buffer for token tile bn, and whether the
// block size is one the kernel takes (0, 32, 64 or >= 128).
cudaError_t prepare_ffn_tc_decode();
bool tc_decode_fits(int64_t K, int splits, int bn, int block_size);
cudaError_t launch_ffn_tc_decode(const FfnArgs& a, int bn, int32_t* status, cudaStream_t st);
cudaError_t launch_gather_rows(const void* x, const int32_t* perm, void* xp, int64_t R, int64_t row_bytes,
                               cudaStream_t st);
// The same gather with each routed row scaled by its router weight
// (apply_router_weight_on_input), rounded to the activation dtype.
cudaError_t launch_gather_rows_weighted(const void* x, const int32_t* perm, const int32_t* inv,
                                        const float* topk_w, int k, void* xp, int64_t R, int64_t H, int act_bf16,
                                        cudaStream_t st);

// Int8 block compute tier: per-block int8 rounding of activation rows (layout
// of the codes: 0 natural, 1 the 4-code order of 4-bit weights for the
// streaming kernel, 2 / 3 the tensor-core order for 4- / 8-bit weights), and
// the expert FFN layer on the codes.
cudaError_t launch_quantize_i8(const void* x, int act_bf16, int64_t rows, int64_t K, int bs, int layout, int8_t* q,
                               float* s, cudaStream_t st);
int64_t i8_smem_bytes(int64_t K, int bits, int block_size, int splits, int nt);
cudaError_t prepare_ffn_i8();
cudaError_t launch_ffn_i8(const FfnArgs& a, cudaStream_t st);
// Router-weighted combine with fc2 bias and shared output; sums the FC2
// split partials in fixed order.
struct CombineArgs {
    const float* o;          // [splits, R, H]
    const int32_t* topk_idx;
    const float* topk_w;
    const int32_t* inv;
    const float* b2;         // [E, H] or nullptr
    const void* shared;      // [T, H] or nullptr
    void* y;                 // [T, H]
    int64_t T, H, R;
    int k, splits, act_bf16;
    float rsf;               // routed_scaling_factor (1 when unset)
    int weights_on_input;    // the router weights already scaled FC1's input rows
    int pdl;                 // launched as a programmatic dependent of FC2
};
cudaError_t launch_combine(const CombineArgs& a, cudaStream_t st);

}  // namespace qmoe
