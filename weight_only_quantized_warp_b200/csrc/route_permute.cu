// route_permute.cu -- top-k softmax routing and the token -> expert
// permutation.
//
// Routing follows the "MoE" page (clika_runtime.nn) class summary -- a router
// picks the top-k experts per token and the outputs combine under the router
// weights -- with the QMoE page's k and normalize_routing_weights attributes.
// Readings: selection is by raw logit (exact in any precision, so the
// selection is bit-identical to any other exact implementation), ties go to
// the lower expert id, and the list is ordered by (logit descending, id
// ascending); a NaN logit reads as -inf. The weights are the softmax over all E logits restricted to the
// selection, renormalised over the k when asked.
//
// The permutation groups the T*k (token, slot) pairs into per-expert
// segments, experts ascending and tokens ascending inside a segment: the
// order in which the "per-expert kernels" ("ClikaRT::nn::QMoEWoQ", class
// description) consume their rows.
#include "qmoe_internal.cuh"

namespace qmoe {
namespace {

constexpr int kMaxPerLane = 8;  // E <= 256

__device__ __forceinline__ bool better(float v, int e, float bv, int be) {
    return v > bv || (v == bv && e < be);
}

// Route token t with one warp (lane = this thread's lane). With n_group > 1
// the experts form n_group consecutive groups; only the topk_group groups of
// largest member logit (ties to the lower group id) may be selected.
// sbias (nullable): the e_score_correction_bias. It moves the selection
// only: experts and groups are ranked by the key fp32(logit + bias), the
// weights stay the softmax of the unbiased logits.
__device__ __forceinline__ void route_token(const void* logits, int act_bf16, int64_t t, int E, int k,
                                            int normalize, int n_group, int topk_group,
                                            const float* __restrict__ sbias,
                                            int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
                                            int lane) {
    float v[kMaxPerLane];   // selection keys
    float lv[kMaxPerLane];  // logits
    const int per = (E + 31) >> 5;
#pragma unroll
    for (int i = 0; i < kMaxPerLane; ++i) {
        const int e = lane + 32 * i;
        v[i] = lv[i] = 0.0f;
        if (i < per && e < E) {
            lv[i] = act_bf16 ? __bfloat162float(((const __nv_bfloat16*)logits)[t * E + e])
                             : ((const float*)logits)[t * E + e];
            // a NaN logit never wins a comparison; read as -inf it still
            // loses to every number and ties resolve by id, so every
            // selected index is a real expert
            if (isnan(lv[i])) lv[i] = -INFINITY;
            v[i] = sbias ? __fadd_rn(lv[i], sbias[e]) : lv[i];
            if (isnan(v[i])) v[i] = -INFINITY;
        }
    }
    // max over all E
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < kMaxPerLane; ++i)
        if (i < per && lane + 32 * i < E) mx = fmaxf(mx, lv[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    // softmax numerators and denominator over all E (fixed reduction tree)
    float ex[kMaxPerLane];
    float z = 0.0f;
#pragma unroll
    for (int i = 0; i < kMaxPerLane; ++i) {
        ex[i] = 0.0f;
        if (i < per && lane + 32 * i < E) {
            ex[i] = expf(lv[i] - mx);
            z += ex[i];
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);

    // allowed slots (bit i: expert lane + 32 i may be selected)
    uint32_t allow = 0xffffffffu;
    if (n_group > 1) {
        const int gsize = E / n_group;
        float gmax = -INFINITY;  // lane g: largest logit of group g
        for (int g = 0; g < n_group; ++g) {
            float m = -INFINITY;
#pragma unroll
            for (int i = 0; i < kMaxPerLane; ++i) {
                const int e = lane + 32 * i;
                if (i < per && e < E && e / gsize == g) m = fmaxf(m, v[i]);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            if (lane == g) gmax = m;
        }
        uint32_t kept = 0;
        for (int r = 0; r < topk_group; ++r) {
            float bv = (lane < n_group && !((kept >> lane) & 1u)) ? gmax : -INFINITY;
            int bg = (lane < n_group && !((kept >> lane) & 1u)) ? lane : 0x7fffffff;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                const int og = __shfl_xor_sync(0xffffffffu, bg, o);
                if (better(ov, og, bv, bg)) {
                    bv = ov;
                    bg = og;
                }
            }
            kept |= 1u << bg;
        }
        allow = 0;
#pragma unroll
        for (int i = 0; i < kMaxPerLane; ++i) {
            const int e = lane + 32 * i;
            if (i < per && e < E && ((kept >> (e / gsize)) & 1u)) allow |= 1u << i;
        }
    }

    uint32_t taken = 0;
    float p_keep[kMaxPerLane];  // p_j kept by lane j%32 in slot j/32
    float sel = 0.0f;
    for (int j = 0; j < k; ++j) {
        float bv = -INFINITY;
        int be = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < kMaxPerLane; ++i) {
            const int e = lane + 32 * i;
            if (i < per && e < E && ((allow & ~taken) >> i & 1u) && better(v[i], e, bv, be)) {
                bv = v[i];
                be = e;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oe = __shfl_xor_sync(0xffffffffu, be, o);
            if (better(ov, oe, bv, be)) {
                bv = ov;
                be = oe;
            }
        }
        if ((be & 31) == lane) taken |= 1u << (be >> 5);
        // the selected expert's softmax numerator, from the lane that holds it
        float mine = 0.0f;
#pragma unroll
        for (int i = 0; i < kMaxPerLane; ++i)
            if (i == (be >> 5)) mine = ex[i];
        const float p = __shfl_sync(0xffffffffu, mine, be & 31);
        sel += p;
        if ((j & 31) == lane) p_keep[j >> 5] = p;
        if (lane == 0) topk_idx[t * k + j] = be;
    }
    const float den = normalize ? sel : z;
#pragma unroll
    for (int s = 0; s < kMaxPerLane; ++s) {
        const int j = lane + 32 * s;
        if (j < k) topk_w[t * k + j] = p_keep[s] / den;
    }
}

// One warp per token. Thread 0 also clears the workspace status word, which
// no kernel of the forward has written yet.
__global__ void route_kernel(const void* logits, int act_bf16, int64_t T, int E, int k,
                             int normalize, int n_group, int topk_group, const float* __restrict__ sbias,
                             int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
                             int32_t* __restrict__ status) {
    if (blockIdx.x == 0 && threadIdx.x == 0) *status = 0;
    const int64_t t = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    if (t >= T) return;
    route_token(logits, act_bf16, t, E, k, normalize, n_group, topk_group, sbias, topk_idx, topk_w,
                threadIdx.x & 31);
}

// One CTA of 1024 threads. Token chunks of 1024: for each chunk, warp-level
// bit masks per expert give each (token, expert) pair its rank among the
// chunk's earlier tokens; a running per-expert base carries across chunks.
constexpr int kPermThreads = 1024;
constexpr int kWarps = kPermThreads / 32;

__device__ __forceinline__ void permute_block(const int32_t* __restrict__ topk_idx, int64_t T, int E, int k,
                                              int32_t* __restrict__ offsets, int32_t* __restrict__ perm_tok,
                                              int32_t* __restrict__ inv, uint32_t* sm) {
    uint32_t* mask = sm;                   // [kWarps][E]
    uint32_t* wpre = mask + kWarps * E;    // [kWarps][E] exclusive prefix over warps
    int32_t* cnt = (int32_t*)(wpre + kWarps * E);  // [E]
    int32_t* off = cnt + E;                // [E + 1]
    int32_t* base = off + E + 1;           // [E]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t R = T * k;

    for (int e = tid; e < E; e += kPermThreads) {
        cnt[e] = 0;
        base[e] = 0;
    }
    __syncthreads();
    for (int64_t r = tid; r < R; r += kPermThreads) atomicAdd(&cnt[topk_idx[r]], 1);
    __syncthreads();
    if (warp == 0) {  // exclusive scan over E with one warp
        int carry = 0;
        for (int e0 = 0; e0 < E; e0 += 32) {
            const int e = e0 + lane;
            int v = e < E ? cnt[e] : 0;
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += n;
            }
            if (e < E) off[e] = carry + incl - v;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) off[E] = carry;
    }
    __syncthreads();
    for (int e = tid; e <= E; e += kPermThreads) offsets[e] = off[e];

    const uint32_t lt = (1u << lane) - 1u;
    for (int64_t t0 = 0; t0 < T; t0 += kPermThreads) {
        for (int i = tid; i < kWarps * E; i += kPermThreads) mask[i] = 0;
        __syncthreads();
        const int64_t t = t0 + tid;
        if (t < T)
            for (int j = 0; j < k; ++j) atomicOr(&mask[warp * E + topk_idx[t * k + j]], 1u << lane);
        __syncthreads();
        for (int e = tid; e < E; e += kPermThreads) {
            uint32_t run = 0;
            for (int w = 0; w < kWarps; ++w) {
                wpre[w * E + e] = run;
                run += __popc(mask[w * E + e]);
            }
        }
        __syncthreads();
        if (t < T) {
            for (int j = 0; j < k; ++j) {
                const int e = topk_idx[t * k + j];
                const int64_t pos = (int64_t)off[e] + base[e] + wpre[warp * E + e] +
                                    __popc(mask[warp * E + e] & lt);
                perm_tok[pos] = int32_t(t);
                inv[t * k + j] = int32_t(pos);
            }
        }
        __syncthreads();
        for (int e = tid; e < E; e += kPermThreads)
            base[e] += wpre[(kWarps - 1) * E + e] + __popc(mask[(kWarps - 1) * E + e]);
        __syncthreads();
    }
}

__global__ void __launch_bounds__(kPermThreads) permute_kernel(
    const int32_t* __restrict__ topk_idx, int64_t T, int E, int k, int32_t* __restrict__ offsets,
    int32_t* __restrict__ perm_tok, int32_t* __restrict__ inv) {
    extern __shared__ uint32_t sm[];
    pdl_trigger();  // the expert kernels may launch and prefetch weights meanwhile
    permute_block(topk_idx, T, E, k, offsets, perm_tok, inv, sm);
}

// The permutation by one warp (few routed pairs): histogram and scan in
// shared memory, then the pairs in order, 32 at a time; lanes holding the
// same expert find each other with a match and take consecutive slots after
// the expert's running base, so a segment keeps token order.
__device__ __forceinline__ void permute_warp(const int32_t* __restrict__ topk_idx, int64_t T, int E, int k,
                                             int32_t* __restrict__ offsets, int32_t* __restrict__ perm_tok,
                                             int32_t* __restrict__ inv, int32_t* cnt, int32_t* base, int lane) {
    const int R = int(T) * k;
    for (int e = lane; e < E; e += 32) cnt[e] = 0;
    __syncwarp();
    for (int r = lane; r < R; r += 32) atomicAdd(&cnt[topk_idx[r]], 1);
    __syncwarp();
    int carry = 0;
    for (int e0 = 0; e0 < E; e0 += 32) {
        const int e = e0 + lane;
        const int v = e < E ? cnt[e] : 0;
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += n;
        }
        if (e < E) {
            offsets[e] = carry + incl - v;
            base[e] = carry + incl - v;
        }
        carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) offsets[E] = carry;
    __syncwarp();
    const uint32_t lt = (1u << lane) - 1u;
    for (int r0 = 0; r0 < R; r0 += 32) {
        const int r = r0 + lane;
        const uint32_t act = __ballot_sync(0xffffffffu, r < R);
        if (r < R) {
            const int e = topk_idx[r];
            const uint32_t same = __match_any_sync(act, e);
            const int rank = __popc(same & lt);
            const int pos = base[e] + rank;
            perm_tok[pos] = r / k;
            inv[r] = pos;
            __syncwarp(act);  // every lane has read base[e] before it moves on
            if (rank == 0) base[e] += __popc(same);
        }
        __syncwarp();
    }
}

// Few tokens: one CTA routes them (a warp per token) and, after a barrier
// that makes the top-k lists visible to the whole block, one warp permutes
// them; one launch instead of two. Thread 0 clears the workspace status word
// first.
__global__ void __launch_bounds__(kPermThreads) route_permute_kernel(
    const void* logits, int act_bf16, int64_t T, int E, int k, int normalize, int n_group, int topk_group,
    const float* __restrict__ sbias, int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
    int32_t* __restrict__ offsets, int32_t* __restrict__ perm_tok, int32_t* __restrict__ inv,
    int32_t* __restrict__ status) {
    extern __shared__ uint32_t sm[];
    pdl_trigger();  // the expert kernels may launch and prefetch weights meanwhile
    if (threadIdx.x == 0) *status = 0;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int64_t t = warp; t < T; t += kWarps)
        route_token(logits, act_bf16, t, E, k, normalize, n_group, topk_group, sbias, topk_idx, topk_w, lane);
    __syncthreads();
    if (warp == 0) {
        int32_t* cnt = reinterpret_cast<int32_t*>(sm);
        permute_warp(topk_idx, T, E, k, offsets, perm_tok, inv, cnt, cnt + E, lane);
    }
}

}  // namespace

cudaError_t launch_route(const void* logits, int act_bf16, int64_t T, int E, int k, int normalize, int n_group,
                         int topk_group, const float* sbias, int32_t* topk_idx, float* topk_w, int32_t* status,
                         cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    const int threads = 256;
    const int64_t blocks = (T * 32 + threads - 1) / threads;
    route_kernel<<<unsigned(blocks), threads, 0, st>>>(logits, act_bf16, T, E, k, normalize, n_group, topk_group,
                                                       sbias, topk_idx, topk_w, status);
    return cudaGetLastError();
}

size_t permute_smem_bytes(int E) {
    return sizeof(uint32_t) * (2 * kWarps * E) + sizeof(int32_t) * (3 * E + 1);
}

cudaError_t launch_route_permute(const void* logits, int act_bf16, int64_t T, int E, int k, int normalize,
                                 int n_group, int topk_group, const float* sbias, int32_t* topk_idx, float* topk_w,
                                 int32_t* offsets, int32_t* perm_tok, int32_t* inv, int32_t* status,
                                 cudaStream_t st) {
    route_permute_kernel<<<1, kPermThreads, permute_smem_bytes(E), st>>>(
        logits, act_bf16, T, E, k, normalize, n_group, topk_group, sbias, topk_idx, topk_w, offsets, perm_tok, inv,
        status);
    return cudaGetLastError();
}


cudaError_t prepare_route_permute() {
    cudaError_t e = cudaFuncSetAttribute(permute_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(permute_smem_bytes(256)));
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(route_permute_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(permute_smem_bytes(256)));
    return e;
}

cudaError_t launch_permute(const int32_t* topk_idx, int64_t T, int E, int k, int32_t* offsets,
                           int32_t* perm_tok, int32_t* inv, cudaStream_t st) {
    permute_kernel<<<1, kPermThreads, permute_smem_bytes(E), st>>>(topk_idx, T, E, k, offsets,
                                                                  perm_tok, inv);
    return cudaGetLastError();
}

namespace {

__global__ void scatter_row_experts_kernel(const int32_t* __restrict__ topk_idx, const int32_t* __restrict__ inv,
                                           int64_t R, int32_t* __restrict__ row_expert) {
    for (int64_t s = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; s < R; s += int64_t(gridDim.x) * blockDim.x)
        row_expert[inv[s]] = topk_idx[s];
}

__global__ void rebase_experts_kernel(const int32_t* __restrict__ ids, int64_t R, int32_t base, int E,
                                      int32_t* __restrict__ local, int32_t* status) {
    for (int64_t r = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; r < R; r += int64_t(gridDim.x) * blockDim.x) {
        const int64_t e = int64_t(ids[r]) - base;
        const bool ok = e >= 0 && e < E;
        local[r] = ok ? int32_t(e) : 0;
        if (!ok) atomicExch(status, int32_t(QMOE_INVALID_ARGUMENT));
    }
}

int blocks_for(int64_t n) { return int(std::min<int64_t>((n + 255) / 256, 148 * 8)); }

}  // namespace

cudaError_t launch_scatter_row_experts(const int32_t* topk_idx, const int32_t* inv, int64_t R, int32_t* row_expert,
                                       cudaStream_t st) {
    if (R <= 0) return cudaSuccess;
    scatter_row_experts_kernel<<<blocks_for(R), 256, 0, st>>>(topk_idx, inv, R, row_expert);
    return cudaGetLastError();
}

cudaError_t launch_rebase_experts(const int32_t* ids, int64_t R, int32_t base, int E, int32_t* local,
                                  int32_t* status, cudaStream_t st) {
    rebase_experts_kernel<<<std::max(1, blocks_for(R)), 256, 0, st>>>(ids, R, base, E, local, status);
    return cudaGetLastError();
}

}  // namespace qmoe
