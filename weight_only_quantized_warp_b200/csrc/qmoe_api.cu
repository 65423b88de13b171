// qmoe_api.cu -- the C ABI declared in include/qmoe.h: attribute validation,
// the one-time pack, the per-call plan and workspace layout, and the launch
// sequence of the forward. The lifecycle follows "ClikaRT::nn::QMoEWoQ":
// make() declares storage-free slots, set_weights() binds and (here) packs
// once, forward() serves from the pack, ~QMoEWoQ() releases it.
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <new>

#include "qmoe_internal.cuh"

namespace qmoe {

static size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

static int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Resident warps per SM assumed when sizing the FC2 split-K.
static constexpr int64_t kSms = 148;

Plan make_plan(const qmoe_handle& h, int64_t T, bool rows_mode) {
    const qmoe_config& c = h.cfg;
    Plan p;
    p.T = T;
    p.R = rows_mode ? T : T * c.k;
    const bool bf16 = c.act_dtype == QMOE_DTYPE_BF16;
    const int64_t E = c.num_experts, H = c.hidden_size, I = c.inter_size;
    const int bits = c.expert_weight_bits, bs = c.block_size;
    const int64_t per_expert = ceil_div(std::max<int64_t>(p.R, 1), E);
    const int64_t touched = std::min<int64_t>(E, std::max<int64_t>(p.R, 1));
    // streaming decode on the tensor cores: token tile 16 or 32, FC1 unsplit,
    // FC2 split until every SM has work and each split's activations fit
    const int tcd_bn = per_expert <= 16 ? 16 : 32;
    int tcd_s2 = 1;
    const int64_t max_s2 = std::max<int64_t>(1, I / 128);  // every split keeps >= one 128-k stage
    while (tcd_s2 < max_s2 && (!tc_decode_fits(I, tcd_s2, tcd_bn, bs) ||
                               touched * (padded_rows(H) / kBlockRows) * tcd_s2 < 4 * kSms))
        ++tcd_s2;
    const bool tcd_ok = per_expert <= 32 && tc_decode_fits(H, 1, tcd_bn, bs) && tc_decode_fits(I, tcd_s2, tcd_bn, bs);
    if (c.compute_mode == QMOE_COMPUTE_INT8_BLOCK) {
        // the int8 tier: the integer tcgen05 GEMM for bf16 activations where
        // it measured faster than the streaming integer mma.sync kernel -- K
        // blocks of 128 or more (one partial fold per 128 k or fewer) and more
        // than 32 rows per expert; QMOE_OPT_PATH 2 forces it, 1 and 3 the
        // streaming kernel
        const bool tc_ok = bf16 && tc_i8_supports(bits, bs, H, I);
        const bool want_tc = h.path_override == kPathTc ||
                             (h.path_override == -1 && per_expert > 32 && bs >= 128);
        p.path = tc_ok && want_tc ? kPathI8Tc : kPathI8;
    }
    else if (!bf16)
        p.path = kPathSimt;
    else if (h.path_override == kPathDecode || h.path_override == kPathTc)
        p.path = h.path_override;
    else if (h.path_override == kPathTcDecode)
        p.path = tcd_ok ? kPathTcDecode : kPathDecode;
    else
        p.path = per_expert <= kDecodeRowsPerExpert ? kPathDecode : kPathTc;
    if (p.path == kPathTcDecode) {
        p.bn = tcd_bn;
        p.fc2_splits = tcd_s2;
    }
    if (p.path == kPathDecode || p.path == kPathI8) {
        // shared memory of one CTA: staged bf16 rows, or int8 code rows
        auto smem = [&](int64_t K, int splits, int nt) {
            return p.path == kPathI8 ? i8_smem_bytes(K, bits, bs, splits, nt)
                                     : decode_smem_bytes(K, bits, bs, splits, nt);
        };
        p.nt = per_expert <= 8 ? 1 : (per_expert <= 16 ? 2 : 4);
        if (h.decode_tiles > 0) p.nt = h.decode_tiles;
        // FC1 runs unsplit; keep its staged rows small enough for at least two CTAs per SM
        while (p.nt > 1 && smem(H, 1, p.nt) > kDecodeSmemTarget) p.nt /= 2;
        // FC2 split-K: every CTA (one 128-row block of one touched expert and
        // one split) streams the same bytes, so the launch takes about
        // ceil(CTAs / slots) rounds of the resident CTA slots; take the split
        // count (1..8, staged rows within the shared-memory target) whose
        // CTAs fill those rounds best, the fewest splits on a tie
        const int64_t ngr = I / kgroup_of(bits);
        const int64_t slots = kSms * (p.nt == 1 ? 3 : 2);
        const int64_t blocks = touched * (padded_rows(H) / kBlockRows);
        int64_t best = 0;
        double best_eff = -1.0;
        for (int64_t s = 1; s <= std::min<int64_t>(8, ngr); ++s) {
            if (smem(I, int(s), p.nt) > kDecodeSmemTarget) continue;
            const int64_t ctas = blocks * s;
            const double eff = double(ctas) / double(slots * ceil_div(ctas, slots));
            if (eff > best_eff + 1e-9) {
                best_eff = eff;
                best = s;
            }
        }
        if (best == 0) {  // no split count fits the target: the smallest that fits the limit
            best = 1;
            while (best < ngr && smem(I, int(best), p.nt) > kDecodeSmemTarget) ++best;
        }
        p.fc2_splits = int(best);
        p.ok = smem(H, 1, p.nt) <= int64_t(kDecodeSmemLimit) &&
               smem(I, p.fc2_splits, p.nt) <= int64_t(kDecodeSmemLimit);
    } else if (p.path == kPathTc || p.path == kPathI8Tc) {
        // token tile: the power of two covering the average segment with a
        // third to spare, so that most experts take one tile (the weights of
        // an expert are decoded once per tile); at most 64 on the int8 tier,
        // whose fold warps hold a tile's fp32 sums in registers
        const int bnmax = p.path == kPathTc ? 256 : 64;
        int bn = 16;
        while (bn < bnmax && bn < ceil_div(4 * per_expert, 3)) bn *= 2;
        p.bn = bn;
        // FC2 work items: touched experts x 128-row blocks x token tiles;
        // split K until every SM has about two items. The int8 tier's
        // 128-k stages split on K-block boundaries only for blocks up to 128.
        const int64_t items = touched * (padded_rows(H) / kBlockRows) * std::max<int64_t>(1, ceil_div(per_expert, bn));
        const int64_t kstage = p.path == kPathTc ? 64 : 128;
        int64_t s = 1;
        if (p.path == kPathTc || bs <= 128)
            while (items * s < 2 * kSms && s < 8 && s * 2 <= I / kstage) s *= 2;
        p.fc2_splits = int(s);
    }
    p.fused_route = T <= kFusedRouteTokens;
    // the row gather runs on the tensor-core paths, and on every path when
    // the router weights scale the expert inputs
    p.gather = p.path == kPathTc || p.path == kPathTcDecode || p.path == kPathI8Tc ||
               (!rows_mode && c.apply_router_weight_on_input);
    // the int8 tier adds the rounding of FC1's input rows and of h
    const bool i8 = p.path == kPathI8 || p.path == kPathI8Tc;
    p.launches = (p.fused_route ? 1 : 2) + (p.gather ? 1 : 0) + 3 + (i8 ? 2 : 0);
    const size_t R = size_t(p.R);
    const size_t act = bf16 ? 2 : 4;
    size_t off = 0;
    p.off_status = off;  off = align256(off + 16);  // fixed place, independent of T
    p.off_idx = off;     off = align256(off + R * 4);
    p.off_w = off;       off = align256(off + R * 4);
    p.off_inv = off;     off = align256(off + R * 4);
    p.off_perm = off;    off = align256(off + R * 4);
    p.off_offsets = off; off = align256(off + size_t(E + 1) * 4);
    p.off_h = off;       off = align256(off + R * size_t(I) * act);
    p.off_xperm = off;
    off = align256(off + (p.gather ? R * size_t(H) * act : 0));
    p.off_o = off;       off = align256(off + size_t(p.fc2_splits) * R * size_t(H) * 4);
    if (i8) {
        const size_t nsb1 = size_t(H / bs), nsb2 = size_t(I / bs);
        p.xq_rows = p.gather ? p.R : T;
        const size_t xr = size_t(p.xq_rows);
        p.off_xq = off; off = align256(off + xr * size_t(H));
        p.off_xs = off; off = align256(off + xr * nsb1 * 4);
        p.off_hq = off; off = align256(off + R * size_t(I));
        p.off_hs = off; off = align256(off + R * nsb2 * 4);
    }
    p.total = off;
    return p;
}

}  // namespace qmoe

using namespace qmoe;

namespace {

qmoe_status fail(const qmoe_handle* h, qmoe_status s, const char* fmt, ...) {
    if (h) {
        char buf[512];
        va_list ap;
        va_start(ap, fmt);
        vsnprintf(buf, sizeof buf, fmt, ap);
        va_end(ap);
        h->last_error = buf;
    }
    return s;
}

qmoe_status cuda_fail(const qmoe_handle* h, cudaError_t e, const char* where) {
    return fail(h, QMOE_CUDA_ERROR, "%s: %s", where, cudaGetErrorString(e));
}

bool pow2(int64_t v) { return v > 0 && (v & (v - 1)) == 0; }

qmoe_status validate(const qmoe_config& c, std::string& why) {
    char buf[256];
    auto bad = [&](qmoe_status s, const char* msg) {
        why = msg;
        return s;
    };
    if (c.num_experts < 1 || c.hidden_size < 1 || c.inter_size < 1)
        return bad(QMOE_INVALID_ARGUMENT, "num_experts, hidden_size and inter_size must be >= 1");
    if (c.k < 1 || c.k > c.num_experts) return bad(QMOE_INVALID_ARGUMENT, "k must lie in [1, num_experts]");
    if (c.expert_weight_bits != 4 && c.expert_weight_bits != 8)
        return bad(QMOE_INVALID_ARGUMENT, "expert_weight_bits must be 4 or 8");
    if (c.block_size != 0) {
        if (!pow2(c.block_size) || c.block_size < 16)
            return bad(QMOE_INVALID_ARGUMENT, "block_size must be 0 or a power of two >= 16");
        if (c.hidden_size % c.block_size || c.inter_size % c.block_size)
            return bad(QMOE_INVALID_ARGUMENT, "hidden_size and inter_size must divide by block_size");
    }
    if (c.activation_type < QMOE_ACT_RELU || c.activation_type > QMOE_ACT_IDENTITY)
        return bad(QMOE_INVALID_ARGUMENT, "activation_type out of range");
    if (c.swiglu_fusion < 0 || c.swiglu_fusion > 2)
        return bad(QMOE_INVALID_ARGUMENT, "swiglu_fusion must be 0, 1 or 2");
    if (c.has_fc3 && c.swiglu_fusion != 0)
        return bad(QMOE_INVALID_ARGUMENT, "fc3 is only defined with swiglu_fusion 0");
    if (c.has_fc3_bias && !c.has_fc3) return bad(QMOE_INVALID_ARGUMENT, "fc3 bias without an fc3 slot");
    const bool gated = c.swiglu_fusion != 0 || c.has_fc3;
    if (!gated && c.activation_type == QMOE_ACT_SWIGLU)
        return bad(QMOE_INVALID_ARGUMENT, "swiglu needs a gate and an up projection (fusion 1/2 or fc3)");
    if (c.weight_format != QMOE_WEIGHTS_INT && c.weight_format != QMOE_WEIGHTS_MXFP4)
        return bad(QMOE_INVALID_ARGUMENT, "weight_format must be INT or MXFP4");
    if (c.weight_format == QMOE_WEIGHTS_MXFP4) {
        if (c.expert_weight_bits != 4 || c.block_size != 32 || c.scale_dtype != QMOE_DTYPE_E8M0)
            return bad(QMOE_INVALID_ARGUMENT, "MXFP4 needs 4-bit codes, block_size 32 and E8M0 scales");
        if (c.act_dtype != QMOE_DTYPE_F32 && c.act_dtype != QMOE_DTYPE_BF16)
            return bad(QMOE_INVALID_ARGUMENT, "act_dtype must be F32 or BF16");
    } else if ((c.act_dtype != QMOE_DTYPE_F32 && c.act_dtype != QMOE_DTYPE_BF16) ||
               (c.scale_dtype != QMOE_DTYPE_F32 && c.scale_dtype != QMOE_DTYPE_BF16)) {
        return bad(QMOE_INVALID_ARGUMENT, "act_dtype and scale_dtype must be F32 or BF16");
    }
    if (c.reserved != 0) return bad(QMOE_INVALID_ARGUMENT, "reserved fields must be 0");
    if (c.compute_mode != QMOE_COMPUTE_FLOAT && c.compute_mode != QMOE_COMPUTE_INT8_BLOCK)
        return bad(QMOE_INVALID_ARGUMENT, "compute_mode must be FLOAT or INT8_BLOCK");
    if (c.compute_mode == QMOE_COMPUTE_INT8_BLOCK) {
        if (c.weight_format != QMOE_WEIGHTS_INT || c.block_size == 0)
            return bad(QMOE_INVALID_ARGUMENT, "the int8 block tier needs integer codes with block scales");
        if (c.block_size < kgroup_of(c.expert_weight_bits))
            return bad(QMOE_UNSUPPORTED,
                       "int8 block tier: block_size below 64 (4-bit codes) or 32 (8-bit codes) is not built");
    }
    if (c.use_sparse_mixer) return bad(QMOE_UNSUPPORTED, "use_sparse_mixer is not built");
    if (c.num_experts > 256) return bad(QMOE_UNSUPPORTED, "num_experts > 256 is not built");
    if (c.hidden_size % 64 || c.inter_size % 64) {
        snprintf(buf, sizeof buf, "hidden_size (%lld) and inter_size (%lld) must be multiples of 64",
                 (long long)c.hidden_size, (long long)c.inter_size);
        return bad(QMOE_UNSUPPORTED, buf);
    }
    if (c.num_experts * c.k > (int64_t(1) << 20))
        return bad(QMOE_UNSUPPORTED, "num_experts * k too large");
    if (c.n_group < 0) return bad(QMOE_INVALID_ARGUMENT, "n_group must be >= 0");
    if (c.n_group > 1) {
        if (c.num_experts % c.n_group) return bad(QMOE_INVALID_ARGUMENT, "num_experts must divide by n_group");
        if (c.topk_group < 1 || c.topk_group > c.n_group)
            return bad(QMOE_INVALID_ARGUMENT, "topk_group must lie in [1, n_group]");
        if (c.k > int64_t(c.topk_group) * (c.num_experts / c.n_group))
            return bad(QMOE_INVALID_ARGUMENT, "k exceeds the experts of the kept groups");
        if (c.n_group > 32) return bad(QMOE_UNSUPPORTED, "more than 32 expert groups is not built");
    }
    if (c.apply_router_weight_on_input != 0 && c.apply_router_weight_on_input != 1)
        return bad(QMOE_INVALID_ARGUMENT, "apply_router_weight_on_input must be 0 or 1");
    if (!(c.routed_scaling_factor >= 0.0f) || !std::isfinite(c.routed_scaling_factor))
        return bad(QMOE_INVALID_ARGUMENT, "routed_scaling_factor must be finite and >= 0");
    if (!(c.expert_output_scale >= 0.0f) || !std::isfinite(c.expert_output_scale))
        return bad(QMOE_INVALID_ARGUMENT, "expert_output_scale must be finite and >= 0");
    if (c.gelu_mode != QMOE_GELU_ERF && c.gelu_mode != QMOE_GELU_TANH)
        return bad(QMOE_INVALID_ARGUMENT, "gelu_mode must be QMOE_GELU_ERF or QMOE_GELU_TANH");
    return QMOE_OK;
}

void free_pack(uint8_t*& w1, void*& s1, float*& b1, uint8_t*& w2, void*& s2, float*& b2) {
    cudaFree(w1);
    cudaFree(s1);
    cudaFree(b1);
    cudaFree(w2);
    cudaFree(s2);
    cudaFree(b2);
    w1 = nullptr;
    s1 = nullptr;
    b1 = nullptr;
    w2 = nullptr;
    s2 = nullptr;
    b2 = nullptr;
}

float resolved_alpha(float a) { return (a == 0.0f || !std::isfinite(a)) ? 1.0f : a; }
float resolved_limit(float l) { return (std::isfinite(l) && l > 0.0f) ? l : INFINITY; }

}  // namespace

extern "C" {

const char* qmoe_status_string(qmoe_status s) {
    switch (s) {
        case QMOE_OK: return "QMOE_OK";
        case QMOE_INVALID_ARGUMENT: return "QMOE_INVALID_ARGUMENT";
        case QMOE_NOT_BOUND: return "QMOE_NOT_BOUND";
        case QMOE_UNSUPPORTED: return "QMOE_UNSUPPORTED";
        case QMOE_CUDA_ERROR: return "QMOE_CUDA_ERROR";
        case QMOE_TIMEOUT: return "QMOE_TIMEOUT";
        case QMOE_OUT_OF_MEMORY: return "QMOE_OUT_OF_MEMORY";
    }
    return "QMOE_UNKNOWN_STATUS";
}

const char* qmoe_last_error(const qmoe_handle* h) { return h ? h->last_error.c_str() : ""; }

qmoe_status qmoe_create(const qmoe_config* cfg, qmoe_handle** out) {
    if (!cfg || !out) return QMOE_INVALID_ARGUMENT;
    *out = nullptr;
    std::string why;
    const qmoe_status s = validate(*cfg, why);
    if (s != QMOE_OK) return s;
    qmoe_handle* h = new (std::nothrow) qmoe_handle();
    if (!h) return QMOE_OUT_OF_MEMORY;
    h->cfg = *cfg;
    h->gated = cfg->swiglu_fusion != 0 || cfg->has_fc3;
    h->n1 = (h->gated ? 2 : 1) * cfg->inter_size;
    *out = h;
    return QMOE_OK;
}

void qmoe_destroy(qmoe_handle* h) {
    if (!h) return;
    free_pack(h->w1, h->s1, h->b1, h->w2, h->s2, h->b2);
    cudaFree(h->score_bias);
    delete h;
}

qmoe_status qmoe_set_score_correction_bias(qmoe_handle* h, const void* bias, void* stream) {
    if (!h) return QMOE_INVALID_ARGUMENT;
    std::lock_guard<std::mutex> lock(h->mu);
    if (reinterpret_cast<uintptr_t>(bias) & 3)
        return fail(h, QMOE_INVALID_ARGUMENT, "e_score_correction_bias must be 4-byte aligned");
    if (!bias) {
        cudaFree(h->score_bias);
        h->score_bias = nullptr;
        return QMOE_OK;
    }
    const size_t n = size_t(h->cfg.num_experts) * sizeof(float);
    float* dst = h->score_bias;
    cudaError_t err = cudaSuccess;
    if (!dst && (err = cudaMalloc((void**)&dst, n)) != cudaSuccess) {
        cudaGetLastError();
        return fail(h, QMOE_OUT_OF_MEMORY, "cudaMalloc for e_score_correction_bias: %s", cudaGetErrorString(err));
    }
    cudaStream_t st = (cudaStream_t)stream;
    if ((err = cudaMemcpyAsync(dst, bias, n, cudaMemcpyDeviceToDevice, st)) != cudaSuccess ||
        (err = cudaStreamSynchronize(st)) != cudaSuccess) {
        if (dst != h->score_bias) cudaFree(dst);
        return cuda_fail(h, err, "e_score_correction_bias copy");
    }
    h->score_bias = dst;
    return QMOE_OK;
}

qmoe_status qmoe_set_weights(qmoe_handle* h, const void* fc1_w, const void* fc1_s,
                             const void* fc1_b, const void* fc2_w, const void* fc2_s,
                             const void* fc2_b, const void* fc3_w, const void* fc3_s,
                             const void* fc3_b, void* stream) {
    if (!h) return QMOE_INVALID_ARGUMENT;
    std::lock_guard<std::mutex> lock(h->mu);
    const qmoe_config& c = h->cfg;
    if (!fc1_w || !fc1_s || !fc2_w || !fc2_s)
        return fail(h, QMOE_INVALID_ARGUMENT, "fc1/fc2 weights and scales are required");
    if (bool(fc1_b) != bool(c.has_fc1_bias))
        return fail(h, QMOE_INVALID_ARGUMENT, "fc1 bias must be given iff has_fc1_bias");
    if (bool(fc2_b) != bool(c.has_fc2_bias))
        return fail(h, QMOE_INVALID_ARGUMENT, "fc2 bias must be given iff has_fc2_bias");
    if ((bool(fc3_w) || bool(fc3_s)) != bool(c.has_fc3) || (c.has_fc3 && (!fc3_w || !fc3_s)))
        return fail(h, QMOE_INVALID_ARGUMENT, "fc3 weights and scales must be given iff has_fc3");
    if (bool(fc3_b) != bool(c.has_fc3_bias))
        return fail(h, QMOE_INVALID_ARGUMENT, "fc3 bias must be given iff has_fc3_bias");
    {
        // the pack reads codes byte by byte, scales and biases element by element
        const uintptr_t s_align = c.scale_dtype == QMOE_DTYPE_F32 ? 4 : (c.scale_dtype == QMOE_DTYPE_BF16 ? 2 : 1);
        const uintptr_t b_align = c.act_dtype == QMOE_DTYPE_F32 ? 4 : 2;
        auto addr = [](const void* p) { return reinterpret_cast<uintptr_t>(p); };
        if ((addr(fc1_s) | addr(fc2_s) | addr(fc3_s)) & (s_align - 1))
            return fail(h, QMOE_INVALID_ARGUMENT, "scales must be aligned to their element size");
        if ((addr(fc1_b) | addr(fc2_b) | addr(fc3_b)) & (b_align - 1))
            return fail(h, QMOE_INVALID_ARGUMENT, "biases must be aligned to their element size");
    }

    cudaStream_t st = (cudaStream_t)stream;
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return cuda_fail(h, err, "cudaGetDevice");
    err = prepare_route_permute();
    if (err == cudaSuccess) err = prepare_ffn_decode();
    if (err == cudaSuccess) err = prepare_ffn_tc();
    if (err == cudaSuccess) err = prepare_ffn_i8();
    if (err == cudaSuccess) err = prepare_ffn_tc_i8();
    if (err != cudaSuccess) return cuda_fail(h, err, "prepare kernels");

    const int64_t E = c.num_experts, H = c.hidden_size, I = c.inter_size, N1 = h->n1;
    const int bits = c.expert_weight_bits, bs = c.block_size;
    // packed scales: bf16 or fp32 as given; E8M0 bytes widen to bf16 (exact)
    const size_t ssz = c.scale_dtype == QMOE_DTYPE_F32 ? 4 : 2;
    const int64_t nsb1 = bs ? H / bs : 1, nsb2 = bs ? I / bs : 1;
    const bool any_b1 = c.has_fc1_bias || c.has_fc3_bias;

    uint8_t *w1 = nullptr, *w2 = nullptr;
    void *s1 = nullptr, *s2 = nullptr;
    float *b1 = nullptr, *b2 = nullptr;
    auto alloc = [&](void** p, size_t n) { return cudaMalloc(p, n < 16 ? 16 : n); };
    const int64_t P1 = padded_rows(N1), P2 = padded_rows(H);
    if ((err = alloc((void**)&w1, size_t(E * P1 * H * bits / 8))) != cudaSuccess ||
        (err = alloc(&s1, size_t(E * P1 * nsb1) * ssz)) != cudaSuccess ||
        (any_b1 && (err = alloc((void**)&b1, size_t(E * N1) * 4)) != cudaSuccess) ||
        (err = alloc((void**)&w2, size_t(E * P2 * I * bits / 8))) != cudaSuccess ||
        (err = alloc(&s2, size_t(E * P2 * nsb2) * ssz)) != cudaSuccess ||
        (c.has_fc2_bias && (err = alloc((void**)&b2, size_t(E * H) * 4)) != cudaSuccess)) {
        free_pack(w1, s1, b1, w2, s2, b2);
        cudaGetLastError();
        return fail(h, QMOE_OUT_OF_MEMORY, "cudaMalloc for the pack: %s", cudaGetErrorString(err));
    }

    PackArgs p1{};
    p1.src = (const uint8_t*)fc1_w;
    p1.s_src = fc1_s;
    p1.b_src = fc1_b;
    p1.src_up = (const uint8_t*)fc3_w;
    p1.s_src_up = fc3_s;
    p1.b_src_up = fc3_b;
    p1.dst = w1;
    p1.s_dst = s1;
    p1.b_dst = b1;
    p1.E = E;
    p1.N = N1;
    p1.K = H;
    p1.I = I;
    p1.bits = bits;
    p1.block_size = bs;
    p1.mode = c.has_fc3 ? 3 : c.swiglu_fusion;  // 0 identity, 1 interleaved, 2 concatenated
    p1.scale_bf16 = c.scale_dtype != QMOE_DTYPE_F32;
    p1.scale_e8m0 = c.scale_dtype == QMOE_DTYPE_E8M0;
    p1.act_bf16 = c.act_dtype == QMOE_DTYPE_BF16;
    PackArgs p2 = p1;
    p2.src = (const uint8_t*)fc2_w;
    p2.s_src = fc2_s;
    p2.b_src = fc2_b;
    p2.src_up = nullptr;
    p2.s_src_up = nullptr;
    p2.b_src_up = nullptr;
    p2.dst = w2;
    p2.s_dst = s2;
    p2.b_dst = b2;
    p2.N = H;
    p2.K = I;
    p2.mode = 0;
    if ((err = launch_pack(p1, st)) != cudaSuccess || (err = launch_pack(p2, st)) != cudaSuccess ||
        (err = cudaStreamSynchronize(st)) != cudaSuccess) {
        free_pack(w1, s1, b1, w2, s2, b2);
        return cuda_fail(h, err, "pack");
    }
    free_pack(h->w1, h->s1, h->b1, h->w2, h->s2, h->b2);
    h->w1 = w1;
    h->s1 = s1;
    h->b1 = b1;
    h->w2 = w2;
    h->s2 = s2;
    h->b2 = b2;
    h->device = dev;
    h->bound = true;
    h->last_error.clear();
    return QMOE_OK;
}

qmoe_status qmoe_set_option(qmoe_handle* h, int32_t option, int64_t value) {
    if (!h) return QMOE_INVALID_ARGUMENT;
    if (option == QMOE_OPT_PATH) {
        if (value != -1 && value != kPathDecode && value != kPathTc && value != kPathTcDecode)
            return fail(h, QMOE_INVALID_ARGUMENT, "QMOE_OPT_PATH must be -1, 1, 2 or 3");
        h->path_override = int(value);
        return QMOE_OK;
    }
    if (option == QMOE_OPT_WAIT_LIMIT_NS) {
        if (value < 100000 || value > int64_t(60) * 1000000000)
            return fail(h, QMOE_INVALID_ARGUMENT, "QMOE_OPT_WAIT_LIMIT_NS must lie in [1e5, 6e10] ns");
        h->wait_limit_ns = uint64_t(value);
        return QMOE_OK;
    }
    if (option == QMOE_OPT_PDL) {
        if (value != 0 && value != 1) return fail(h, QMOE_INVALID_ARGUMENT, "QMOE_OPT_PDL must be 0 or 1");
        h->pdl = int(value);
        return QMOE_OK;
    }
    if (option == QMOE_OPT_DECODE_TILES) {
        if (value != 0 && value != 1 && value != 2 && value != 4)
            return fail(h, QMOE_INVALID_ARGUMENT, "QMOE_OPT_DECODE_TILES must be 0, 1, 2 or 4");
        h->decode_tiles = int(value);
        return QMOE_OK;
    }
    if (option == QMOE_OPT_TEST_WITHHOLD) {
        if (value != 0 && value != 1) return fail(h, QMOE_INVALID_ARGUMENT, "QMOE_OPT_TEST_WITHHOLD must be 0 or 1");
        h->withhold = int(value);
        return QMOE_OK;
    }
    return fail(h, QMOE_INVALID_ARGUMENT, "unknown option %d", int(option));
}

size_t qmoe_workspace_size(const qmoe_handle* h, int64_t T) {
    if (!h || T < 0) return 0;
    return make_plan(*h, T).total;
}

int32_t qmoe_path_for(const qmoe_handle* h, int64_t T) {
    if (!h || T < 0) return -1;
    return make_plan(*h, T).path;
}

int32_t qmoe_launches_for(const qmoe_handle* h, int64_t T) {
    if (!h || T < 0) return -1;
    return T == 0 ? 0 : make_plan(*h, T).launches;
}

int32_t qmoe_token_tile_for(const qmoe_handle* h, int64_t T) {
    if (!h || T < 0) return -1;
    const Plan p = make_plan(*h, T);
    return (p.path == kPathTc || p.path == kPathTcDecode || p.path == kPathI8Tc) ? p.bn : 0;
}

}  // extern "C"

// FC1 (+ activation) and FC2 of the routed rows: the row gather where the
// plan wants it, the int8 tier's rounding launches, then the two expert
// layers into the workspace (h, and FC2's fp32 split partials). Shared by
// the whole forward and the expert-parallel rows entry.
template <class Mark>
static cudaError_t ffn_layers(const qmoe_handle* h, const Plan& p, const void* x, int32_t* perm, int32_t* inv,
                              float* tw, int k, bool weighted_rows, char* ws, int32_t* status, cudaStream_t st,
                              Mark& mark, const char** where) {
    const qmoe_config& c = h->cfg;
    const int E = int(c.num_experts);
    const int bf16 = c.act_dtype == QMOE_DTYPE_BF16;
    int32_t* offsets = (int32_t*)(ws + p.off_offsets);
    void* hid = ws + p.off_h;
    float* o = (float*)(ws + p.off_o);
    cudaError_t err;
    FfnArgs f1{};
    f1.W = h->w1;
    f1.S = h->s1;
    f1.bias = h->b1;
    f1.act = x;
    f1.rowmap = perm;
    f1.offsets = offsets;
    f1.out = hid;
    f1.N = h->n1;
    f1.K = c.hidden_size;
    f1.R = p.R;
    f1.E = E;
    f1.bits = c.expert_weight_bits;
    f1.block_size = c.block_size;
    f1.gated = h->gated;
    f1.is_fc1 = 1;
    f1.act_type = (c.activation_type == QMOE_ACT_GELU && c.gelu_mode == QMOE_GELU_TANH) ? kActGeluTanh
                                                                                       : c.activation_type;
    f1.alpha = resolved_alpha(c.activation_alpha);
    f1.beta = c.activation_beta;
    f1.limit = resolved_limit(c.swiglu_limit);
    f1.splits = 1;
    f1.scale_bf16 = c.scale_dtype != QMOE_DTYPE_F32;
    f1.fp4 = c.weight_format == QMOE_WEIGHTS_MXFP4;
    f1.act_bf16 = bf16;
    f1.nt = p.nt;
    f1.timeout_ns = h->wait_limit_ns;
    f1.withhold = h->withhold;
    // the weight-streaming kernels prefetch their first weights while the
    // kernel before them finishes (routing / gather before FC1, FC1 before FC2)
    f1.pdl = h->pdl && p.path == kPathDecode;
    FfnArgs f2 = f1;
    f2.W = h->w2;
    f2.S = h->s2;
    f2.bias = nullptr;
    f2.act = hid;
    f2.rowmap = nullptr;
    f2.out = o;
    f2.N = c.hidden_size;
    f2.K = c.inter_size;
    f2.gated = 0;
    f2.is_fc1 = 0;
    f2.splits = p.fc2_splits;
    if (p.gather) {
        if ((err = mark()) != cudaSuccess) { *where = "event"; return err; }
        void* xp = ws + p.off_xperm;
        err = weighted_rows
                  ? launch_gather_rows_weighted(x, perm, inv, tw, k, xp, p.R, c.hidden_size, bf16, st)
                  : launch_gather_rows(x, perm, xp, p.R, c.hidden_size * 2, st);
        if (err != cudaSuccess) { *where = "gather"; return err; }
        f1.act = xp;
        f1.rowmap = nullptr;  // rows already in segment order
    }
    if (p.path == kPathI8 || p.path == kPathI8Tc) {
        // FC1's input rows (x by token, or the gathered rows) to int8 codes,
        // in the order the chosen kernel reads them
        const bool tc = p.path == kPathI8Tc;
        const int perm = tc ? (c.expert_weight_bits == 4 ? 2 : 3) : (c.expert_weight_bits == 4 ? 1 : 0);
        int8_t* xq = (int8_t*)(ws + p.off_xq);
        float* xs = (float*)(ws + p.off_xs);
        if ((err = mark()) != cudaSuccess) { *where = "event"; return err; }
        if ((err = launch_quantize_i8(f1.act, bf16, p.xq_rows, c.hidden_size, c.block_size, perm, xq, xs, st)) !=
            cudaSuccess)
            { *where = "quantize x"; return err; }
        f1.aq = xq;
        f1.as = xs;
        if ((err = mark()) != cudaSuccess) { *where = "event"; return err; }
        if ((err = tc ? launch_ffn_tc_i8(f1, p.bn, status, st) : launch_ffn_i8(f1, st)) != cudaSuccess)
            { *where = "fc1"; return err; }
        int8_t* hq = (int8_t*)(ws + p.off_hq);
        float* hs = (float*)(ws + p.off_hs);
        if ((err = mark()) != cudaSuccess) { *where = "event"; return err; }
        if ((err = launch_quantize_i8(hid, bf16, p.R, c.inter_size, c.block_size, perm, hq, hs, st)) != cudaSuccess)
            { *where = "quantize h"; return err; }
        f2.aq = hq;
        f2.as = hs;
        if ((err = mark()) != cudaSuccess) { *where = "event"; return err; }
        if ((err = tc ? launch_ffn_tc_i8(f2, p.bn, status, st) : launch_ffn_i8(f2, st)) != cudaSuccess)
            { *where = "fc2"; return err; }
    } else {
        if ((err = mark()) != cudaSuccess) { *where = "event"; return err; }
        err = p.path == kPathSimt        ? launch_ffn_simt(f1, st)
              : p.path == kPathTc        ? launch_ffn_tc(f1, p.bn, status, st)
              : p.path == kPathTcDecode  ? launch_ffn_tc_decode(f1, p.bn, status, st)
                                         : launch_ffn_decode(f1, st);
        if (err != cudaSuccess) { *where = "fc1"; return err; }
        if ((err = mark()) != cudaSuccess) { *where = "event"; return err; }
        err = p.path == kPathSimt        ? launch_ffn_simt(f2, st)
              : p.path == kPathTc        ? launch_ffn_tc(f2, p.bn, status, st)
              : p.path == kPathTcDecode  ? launch_ffn_tc_decode(f2, p.bn, status, st)
                                         : launch_ffn_decode(f2, st);
        if (err != cudaSuccess) { *where = "fc2"; return err; }
    }
    return cudaSuccess;
}

static qmoe_status forward_impl(const qmoe_handle* h, int64_t T, const void* x,
                                const void* router_logits, const void* shared_output, void* y,
                                void* workspace, size_t workspace_bytes, void* stream,
                                void* const* events, int32_t n_events) {
    if (!h) return QMOE_INVALID_ARGUMENT;
    if (T < 0) return fail(h, QMOE_INVALID_ARGUMENT, "T must be >= 0");
    if (T > 0) {
        // the kernels read x and shared_output and write y in 8- and 16-byte
        // vectors, and the logits element by element
        auto addr = [](const void* p) { return reinterpret_cast<uintptr_t>(p); };
        const uintptr_t act_bytes = h->cfg.act_dtype == QMOE_DTYPE_BF16 ? 2 : 4;
        if (!x || !router_logits || !y || !workspace)
            return fail(h, QMOE_INVALID_ARGUMENT, "x, router_logits, y and workspace are required");
        if ((addr(x) | addr(y) | addr(shared_output)) & 15)
            return fail(h, QMOE_INVALID_ARGUMENT, "x, shared_output and y must be 16-byte aligned");
        if (addr(router_logits) & (act_bytes - 1))
            return fail(h, QMOE_INVALID_ARGUMENT, "router_logits must be aligned to its element size");
        if (addr(workspace) & 255) return fail(h, QMOE_INVALID_ARGUMENT, "workspace must be 256-byte aligned");
    }
    if (!h->bound) return fail(h, QMOE_NOT_BOUND, "forward before set_weights bound the weights");
    if (T == 0) return QMOE_OK;
    if (T * h->cfg.k >= (int64_t(1) << 31))
        return fail(h, QMOE_UNSUPPORTED, "T * k must stay below 2^31");
    const Plan p = make_plan(*h, T);
    if (!p.ok)
        return fail(h, QMOE_UNSUPPORTED, "no kernel configuration fits this shape (hidden_size too large)");
    if (workspace_bytes < p.total)
        return fail(h, QMOE_INVALID_ARGUMENT, "workspace too small: %zu < %zu", workspace_bytes,
                    p.total);
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != h->device)
        return fail(h, QMOE_INVALID_ARGUMENT, "current device %d is not the device the weights live on (%d)",
                    dev, h->device);
    const qmoe_config& c = h->cfg;
    cudaStream_t st = (cudaStream_t)stream;
    if (events && n_events != p.launches + 1)
        return fail(h, QMOE_INVALID_ARGUMENT, "n_events must be %d", p.launches + 1);
    int ev_i = 0;
    auto mark = [&]() -> cudaError_t {
        if (!events) return cudaSuccess;
        return cudaEventRecord((cudaEvent_t)events[ev_i++], st);
    };
    char* ws = (char*)workspace;
    int32_t* idx = (int32_t*)(ws + p.off_idx);
    float* tw = (float*)(ws + p.off_w);
    int32_t* inv = (int32_t*)(ws + p.off_inv);
    int32_t* perm = (int32_t*)(ws + p.off_perm);
    int32_t* offsets = (int32_t*)(ws + p.off_offsets);
    void* hid = ws + p.off_h;
    float* o = (float*)(ws + p.off_o);
    const int E = int(c.num_experts), k = int(c.k);
    const int bf16 = c.act_dtype == QMOE_DTYPE_BF16;
    cudaError_t err;
    int32_t* status = (int32_t*)(ws + p.off_status);  // cleared by the first kernel
    if ((err = mark()) != cudaSuccess) return cuda_fail(h, err, "event");
    if (p.fused_route) {
        if ((err = launch_route_permute(router_logits, bf16, T, E, k, c.normalize_routing_weights, c.n_group,
                                        c.topk_group, h->score_bias, idx, tw, offsets, perm, inv, status, st)) !=
            cudaSuccess)
            return cuda_fail(h, err, "route+permute");
    } else {
        if ((err = launch_route(router_logits, bf16, T, E, k, c.normalize_routing_weights, c.n_group, c.topk_group,
                                h->score_bias, idx, tw, status, st)) != cudaSuccess)
            return cuda_fail(h, err, "route");
        if ((err = mark()) != cudaSuccess) return cuda_fail(h, err, "event");
        if ((err = launch_permute(idx, T, E, k, offsets, perm, inv, st)) != cudaSuccess)
            return cuda_fail(h, err, "permute");
    }

    const char* where = "";
    if ((err = ffn_layers(h, p, x, perm, inv, tw, k, c.apply_router_weight_on_input != 0, ws, status, st, mark,
                          &where)) != cudaSuccess)
        return cuda_fail(h, err, where);
    CombineArgs ca{};
    ca.o = o;
    ca.topk_idx = idx;
    ca.topk_w = tw;
    ca.inv = inv;
    ca.b2 = h->b2;
    ca.shared = shared_output;
    ca.y = y;
    ca.T = T;
    ca.H = c.hidden_size;
    ca.R = p.R;
    ca.k = k;
    ca.splits = p.fc2_splits;
    // the routed sum's multiplier: routed_scaling_factor times
    // expert_output_scale (each 0 reads as 1); both scale the expert outputs
    // linearly, so one fp32 product applies them
    ca.rsf = (c.routed_scaling_factor > 0.0f ? c.routed_scaling_factor : 1.0f) *
             (c.expert_output_scale > 0.0f ? c.expert_output_scale : 1.0f);
    ca.weights_on_input = c.apply_router_weight_on_input;
    ca.pdl = h->pdl;
    ca.act_bf16 = bf16;
    if ((err = mark()) != cudaSuccess) return cuda_fail(h, err, "event");
    if ((err = launch_combine(ca, st)) != cudaSuccess) return cuda_fail(h, err, "combine");
    if ((err = mark()) != cudaSuccess) return cuda_fail(h, err, "event");
    return QMOE_OK;
}

extern "C" {

qmoe_status qmoe_forward(const qmoe_handle* h, int64_t T, const void* x, const void* router_logits,
                         const void* shared_output, void* y, void* workspace,
                         size_t workspace_bytes, void* stream) {
    return forward_impl(h, T, x, router_logits, shared_output, y, workspace, workspace_bytes,
                        stream, nullptr, 0);
}

qmoe_status qmoe_forward_profiled(const qmoe_handle* h, int64_t T, const void* x,
                                  const void* router_logits, const void* shared_output, void* y,
                                  void* workspace, size_t workspace_bytes, void* stream,
                                  void* const* events, int32_t n_events) {
    if (!events) return fail(h, QMOE_INVALID_ARGUMENT, "events is required");
    return forward_impl(h, T, x, router_logits, shared_output, y, workspace, workspace_bytes,
                        stream, events, n_events);
}

qmoe_status qmoe_debug_routing(const qmoe_handle* h, int64_t T, const void* workspace,
                               int32_t* topk_idx, float* topk_w, int32_t* offsets,
                               int32_t* perm_tok, int32_t* inv, void* stream) {
    if (!h || !workspace || T < 0) return QMOE_INVALID_ARGUMENT;
    const Plan p = make_plan(*h, T);
    const char* ws = (const char*)workspace;
    cudaStream_t st = (cudaStream_t)stream;
    const size_t R = size_t(p.R);
    cudaError_t err = cudaSuccess;
    auto cp = [&](void* dst, size_t off, size_t n) {
        if (dst && n && err == cudaSuccess)
            err = cudaMemcpyAsync(dst, ws + off, n, cudaMemcpyDeviceToDevice, st);
    };
    cp(topk_idx, p.off_idx, R * 4);
    cp(topk_w, p.off_w, R * 4);
    cp(offsets, p.off_offsets, size_t(h->cfg.num_experts + 1) * 4);
    cp(perm_tok, p.off_perm, R * 4);
    cp(inv, p.off_inv, R * 4);
    return err == cudaSuccess ? QMOE_OK : cuda_fail(h, err, "debug_routing");
}

qmoe_status qmoe_debug_hidden(const qmoe_handle* h, int64_t T, const void* workspace, void* hidden,
                              void* stream) {
    if (!h || !workspace || !hidden || T < 0) return QMOE_INVALID_ARGUMENT;
    const Plan p = make_plan(*h, T);
    const size_t act = h->cfg.act_dtype == QMOE_DTYPE_BF16 ? 2 : 4;
    const size_t n = size_t(p.R) * size_t(h->cfg.inter_size) * act;
    if (!n) return QMOE_OK;
    cudaError_t err = cudaMemcpyAsync(hidden, (const char*)workspace + p.off_h, n,
                                      cudaMemcpyDeviceToDevice, (cudaStream_t)stream);
    return err == cudaSuccess ? QMOE_OK : cuda_fail(h, err, "debug_hidden");
}

qmoe_status qmoe_quantize_act_i8(const void* x, int32_t dtype, int64_t rows, int64_t K, int32_t block_size,
                                 int8_t* q, float* scales, void* stream) {
    if (rows < 0 || K < 1 || !pow2(block_size) || block_size < 16 || K % block_size)
        return QMOE_INVALID_ARGUMENT;
    if (dtype != QMOE_DTYPE_F32 && dtype != QMOE_DTYPE_BF16) return QMOE_INVALID_ARGUMENT;
    if (rows == 0) return QMOE_OK;
    if (!x || !q || !scales || (reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(q) & 3) ||
        (reinterpret_cast<uintptr_t>(scales) & 3))
        return QMOE_INVALID_ARGUMENT;
    const cudaError_t err = launch_quantize_i8(x, dtype == QMOE_DTYPE_BF16, rows, K, block_size, 0, q, scales,
                                               (cudaStream_t)stream);
    return err == cudaSuccess ? QMOE_OK : QMOE_CUDA_ERROR;
}

qmoe_status qmoe_read_device_status(const qmoe_handle* h, const void* workspace, void* stream) {
    if (!h || !workspace) return QMOE_INVALID_ARGUMENT;
    const Plan p = make_plan(*h, 0);
    int32_t v = 0;
    cudaError_t err = cudaMemcpyAsync(&v, (const char*)workspace + p.off_status, 4,
                                      cudaMemcpyDeviceToHost, (cudaStream_t)stream);
    if (err == cudaSuccess) err = cudaStreamSynchronize((cudaStream_t)stream);
    if (err != cudaSuccess) return cuda_fail(h, err, "read_device_status");
    return v == 0 ? QMOE_OK : (v == QMOE_INVALID_ARGUMENT ? QMOE_INVALID_ARGUMENT : QMOE_TIMEOUT);
}

// ---------------------------------------------------------------- expert parallel
// The forward split at its two exchange points: routing, permutation and the
// row gather on the rank that owns the tokens (dispatch); the expert layers on
// the rank that owns the experts (rows); the weighted combine back on the
// token owner (combine). The rows in between travel between ranks in the
// dispatch order, which is expert order, so each destination rank's rows are
// one contiguous range.

}  // extern "C"

namespace {

struct EpState {  // routing of one dispatch, kept for its combine
    size_t off_status, off_idx, off_w, off_inv, off_perm, off_offsets, total;
};

EpState ep_state(const qmoe_handle& h, int64_t T) {
    const size_t R = size_t(T) * size_t(h.cfg.k);
    EpState s;
    size_t off = 0;
    s.off_status = off;  off = align256(off + 16);
    s.off_idx = off;     off = align256(off + R * 4);
    s.off_w = off;       off = align256(off + R * 4);
    s.off_inv = off;     off = align256(off + R * 4);
    s.off_perm = off;    off = align256(off + R * 4);
    s.off_offsets = off; off = align256(off + size_t(h.cfg.num_experts + 1) * 4);
    s.total = off;
    return s;
}

bool misaligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) != 0; }

qmoe_status on_device(const qmoe_handle* h) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return fail(h, QMOE_CUDA_ERROR, "no current device");
    if (h->device >= 0 && dev != h->device)  // a routing handle without weights runs on any device
        return fail(h, QMOE_INVALID_ARGUMENT, "current device %d is not the handle's device (%d)", dev, h->device);
    return QMOE_OK;
}

float routed_multiplier(const qmoe_config& c) {
    return (c.routed_scaling_factor > 0.0f ? c.routed_scaling_factor : 1.0f) *
           (c.expert_output_scale > 0.0f ? c.expert_output_scale : 1.0f);
}

}  // namespace

extern "C" {

size_t qmoe_ep_state_bytes(const qmoe_handle* h, int64_t T) {
    if (!h || T < 0) return 0;
    return ep_state(*h, T).total;
}

size_t qmoe_ep_rows_workspace_size(const qmoe_handle* h, int64_t R) {
    if (!h || R < 0) return 0;
    return make_plan(*h, R, true).total;
}

qmoe_status qmoe_ep_dispatch(const qmoe_handle* h, int64_t T, const void* x, const void* router_logits,
                             void* rows, int32_t* row_expert, int32_t* offsets, void* state, size_t state_bytes,
                             void* stream) {
    if (!h) return QMOE_INVALID_ARGUMENT;
    if (T < 0) return fail(h, QMOE_INVALID_ARGUMENT, "T must be >= 0");
    if (T == 0) return QMOE_OK;
    const qmoe_config& c = h->cfg;
    const int bf16 = c.act_dtype == QMOE_DTYPE_BF16;
    if (!x || !router_logits || !rows || !row_expert || !offsets || !state)
        return fail(h, QMOE_INVALID_ARGUMENT, "x, router_logits, rows, row_expert, offsets and state are required");
    if (misaligned(x, 16) || misaligned(rows, 16) || misaligned(router_logits, bf16 ? 2 : 4) ||
        misaligned(row_expert, 4) || misaligned(offsets, 4) || misaligned(state, 256))
        return fail(h, QMOE_INVALID_ARGUMENT, "x and rows 16-byte, state 256-byte, the rest element aligned");
    if (T * c.k >= (int64_t(1) << 31)) return fail(h, QMOE_UNSUPPORTED, "T * k must stay below 2^31");
    const EpState es = ep_state(*h, T);
    if (state_bytes < es.total)
        return fail(h, QMOE_INVALID_ARGUMENT, "state too small: %zu < %zu", state_bytes, es.total);
    if (qmoe_status s = on_device(h)) return s;
    char* sb = (char*)state;
    int32_t* status = (int32_t*)(sb + es.off_status);
    int32_t* idx = (int32_t*)(sb + es.off_idx);
    float* tw = (float*)(sb + es.off_w);
    int32_t* inv = (int32_t*)(sb + es.off_inv);
    int32_t* perm = (int32_t*)(sb + es.off_perm);
    int32_t* offs = (int32_t*)(sb + es.off_offsets);
    const int E = int(c.num_experts), k = int(c.k);
    const int64_t R = T * k;
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t err;
    if (T <= kFusedRouteTokens)
        err = launch_route_permute(router_logits, bf16, T, E, k, c.normalize_routing_weights, c.n_group,
                                   c.topk_group, h->score_bias, idx, tw, offs, perm, inv, status, st);
    else if ((err = launch_route(router_logits, bf16, T, E, k, c.normalize_routing_weights, c.n_group,
                                 c.topk_group, h->score_bias, idx, tw, status, st)) == cudaSuccess)
        err = launch_permute(idx, T, E, k, offs, perm, inv, st);
    if (err != cudaSuccess) return cuda_fail(h, err, "ep route");
    err = c.apply_router_weight_on_input
              ? launch_gather_rows_weighted(x, perm, inv, tw, k, rows, R, c.hidden_size, bf16, st)
              : launch_gather_rows(x, perm, rows, R, c.hidden_size * (bf16 ? 2 : 4), st);
    if (err == cudaSuccess) err = launch_scatter_row_experts(idx, inv, R, row_expert, st);
    if (err == cudaSuccess)
        err = cudaMemcpyAsync(offsets, offs, size_t(E + 1) * 4, cudaMemcpyDeviceToDevice, st);
    return err == cudaSuccess ? QMOE_OK : cuda_fail(h, err, "ep dispatch");
}

qmoe_status qmoe_ep_expert_rows(const qmoe_handle* h, int64_t R, const void* rows, const int32_t* row_expert,
                                int32_t expert_base, float* out, void* workspace, size_t workspace_bytes,
                                void* stream) {
    if (!h) return QMOE_INVALID_ARGUMENT;
    if (R < 0) return fail(h, QMOE_INVALID_ARGUMENT, "R must be >= 0");
    if (!h->bound) return fail(h, QMOE_NOT_BOUND, "expert rows before set_weights bound the weights");
    if (R == 0) return QMOE_OK;
    if (!rows || !row_expert || !out || !workspace)
        return fail(h, QMOE_INVALID_ARGUMENT, "rows, row_expert, out and workspace are required");
    if (misaligned(rows, 16) || misaligned(out, 16) || misaligned(row_expert, 4) || misaligned(workspace, 256))
        return fail(h, QMOE_INVALID_ARGUMENT, "rows and out 16-byte, workspace 256-byte, row_expert 4-byte aligned");
    if (R >= (int64_t(1) << 31)) return fail(h, QMOE_UNSUPPORTED, "R must stay below 2^31");
    const Plan p = make_plan(*h, R, true);
    if (!p.ok) return fail(h, QMOE_UNSUPPORTED, "no kernel configuration fits this shape (hidden_size too large)");
    if (workspace_bytes < p.total)
        return fail(h, QMOE_INVALID_ARGUMENT, "workspace too small: %zu < %zu", workspace_bytes, p.total);
    if (qmoe_status s = on_device(h)) return s;
    const qmoe_config& c = h->cfg;
    const int E = int(c.num_experts);
    cudaStream_t st = (cudaStream_t)stream;
    char* ws = (char*)workspace;
    int32_t* status = (int32_t*)(ws + p.off_status);
    int32_t* idx = (int32_t*)(ws + p.off_idx);
    float* tw = (float*)(ws + p.off_w);
    int32_t* inv = (int32_t*)(ws + p.off_inv);
    int32_t* perm = (int32_t*)(ws + p.off_perm);
    int32_t* offs = (int32_t*)(ws + p.off_offsets);
    cudaError_t err = cudaMemsetAsync(status, 0, 4, st);
    if (err == cudaSuccess) err = launch_rebase_experts(row_expert, R, expert_base, E, idx, status, st);
    if (err == cudaSuccess) err = launch_permute(idx, R, E, 1, offs, perm, inv, st);
    if (err != cudaSuccess) return cuda_fail(h, err, "ep rows permute");
    auto mark = []() -> cudaError_t { return cudaSuccess; };
    const char* where = "";
    if ((err = ffn_layers(h, p, rows, perm, inv, tw, 1, false, ws, status, st, mark, &where)) != cudaSuccess)
        return cuda_fail(h, err, where);
    // each row's expert output o + b2 in fp32: the combine with one route per
    // row, unit weight and no scaling (the token owner's combine applies them)
    CombineArgs ca{};
    ca.o = (const float*)(ws + p.off_o);
    ca.topk_idx = idx;
    ca.topk_w = tw;
    ca.inv = inv;
    ca.b2 = h->b2;
    ca.shared = nullptr;
    ca.y = out;
    ca.T = R;
    ca.H = c.hidden_size;
    ca.R = p.R;
    ca.k = 1;
    ca.splits = p.fc2_splits;
    ca.rsf = 1.0f;
    ca.weights_on_input = 1;
    ca.pdl = h->pdl;
    ca.act_bf16 = 0;
    if ((err = launch_combine(ca, st)) != cudaSuccess) return cuda_fail(h, err, "ep rows output");
    return QMOE_OK;
}

qmoe_status qmoe_ep_combine(const qmoe_handle* h, int64_t T, const float* expert_out, const void* state,
                            const void* shared_output, void* y, void* stream) {
    if (!h) return QMOE_INVALID_ARGUMENT;
    if (T < 0) return fail(h, QMOE_INVALID_ARGUMENT, "T must be >= 0");
    if (T == 0) return QMOE_OK;
    if (!expert_out || !state || !y)
        return fail(h, QMOE_INVALID_ARGUMENT, "expert_out, state and y are required");
    if (misaligned(expert_out, 16) || misaligned(y, 16) || misaligned(shared_output, 16) || misaligned(state, 256))
        return fail(h, QMOE_INVALID_ARGUMENT, "expert_out, shared_output and y 16-byte, state 256-byte aligned");
    if (qmoe_status s = on_device(h)) return s;
    const qmoe_config& c = h->cfg;
    const EpState es = ep_state(*h, T);
    const char* sb = (const char*)state;
    CombineArgs ca{};
    ca.o = expert_out;
    ca.topk_idx = (const int32_t*)(sb + es.off_idx);
    ca.topk_w = (const float*)(sb + es.off_w);
    ca.inv = (const int32_t*)(sb + es.off_inv);
    ca.b2 = nullptr;  // added with each expert output on the rank that computed it
    ca.shared = shared_output;
    ca.y = y;
    ca.T = T;
    ca.H = c.hidden_size;
    ca.R = T * c.k;
    ca.k = int(c.k);
    ca.splits = 1;
    ca.rsf = routed_multiplier(c);
    ca.weights_on_input = c.apply_router_weight_on_input;
    ca.pdl = 0;
    ca.act_bf16 = c.act_dtype == QMOE_DTYPE_BF16;
    const cudaError_t err = launch_combine(ca, (cudaStream_t)stream);
    return err == cudaSuccess ? QMOE_OK : cuda_fail(h, err, "ep combine");
}

}  // extern "C"
