// common.cuh -- shared device-side definitions of the hybrid attention library.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace hyb {

// Device status flags, kept in the first word of the caller's workspace.
enum : unsigned { FLAG_NONFINITE = 1u, FLAG_TIMEOUT = 2u, FLAG_INTERNAL = 4u };

constexpr int kNumSMs = 148;          // B200
constexpr int kUpdateTile = 128;      // tokens per key-tile of the state update
constexpr size_t kStatusBytes = 256;  // status block at the start of the workspace

// Everything one pass needs; built on the host from the C-ABI arguments.
struct LayerArgs {
    int B, H, T, D;
    int T_kv;              // keys the attention kernel reads (T, or the cached tokens of a KV cache)
    int inter;             // 1: the attention kernel adds O_inter = Q W (hybrid layer); 0: softmax only
    const float* mix;      // [B][H][2] (a, c): out = a O_intra + c O_inter; NULL: a = c = 1
    float sm_scale_log2;   // softmax scale * log2(e)
    float l2_eps;
    const void* q;
    const void* k;
    const void* v;
    const void* phi_q;
    const void* phi_k;
    const void* phi_v;
    const float* gate_logits;
    const float* beta_logits;
    float* state;
    void* out;
    float* out_intra;
    float* out_inter;
    // workspace views
    unsigned* flags;
    float* W;                  // fp32 [BH][D][D]: phi_q^T S (SIMT path)
    __nv_bfloat16* WT_hi;      // bf16 [BH][D][D]: phi_q^T S, row-major, high part (tensor path)
    __nv_bfloat16* WT_lo;      // bf16 [BH][D][D]: low part
    float* S_prev;             // fp32 [BH][D][D]: copy of S_{N-1} (fp32 path, clean pass)
    __nv_bfloat16* w_next;     // if set, the delta update also writes W of the next frame,
                               // phi_q^T S_N, here (hi plane; lo plane BH D^2 further)
    float* partials;           // fp32 [BH][nsplit][D][2D]: per-split [G | P]
    int nsplit;
    int split_tokens;
    // chained passes (tensor path): the delta update lets the next kernel of the
    // stream start at its entry (chain_trigger 1) or once its key tiles are done
    // (chain_trigger 2: the next update of a chain of updates); before reading
    // S_{N-1} it waits until the words chain_flags[bh * 8 + c], c < nsplit, equal
    // chain_wait (0: no wait), which the previous chained update of this state
    // sets once it is done with the state and its W; it sets its own words to
    // chain_set (NULL: no flags)
    unsigned* chain_flags;
    unsigned chain_wait;
    unsigned chain_set;
    int chain_trigger;
    // token-level access: the inter-frame read computed by the token-level kernels,
    // fp32 [B][T][H][D]; the attention kernels add it instead of Q W (NULL: Q W)
    const float* oi_ext;
    // Token Radius Attention: the warm-up pass writes each query's attention entropy
    // (nats, [B][H][T]); a sparse pass walks, for query tile qt of (b, h), the
    // kv_count[bh * n_qt + qt] key blocks listed at kv_list[(bh * n_qt + qt) * kv_stride]
    float* ent_out;
    const int* kv_list;
    const int* kv_count;
    int kv_stride;
    // optional: CTA i of the grid takes query tile row kv_order[i] (bh * n_qt + qt),
    // so the longest lists go first
    const int* kv_order;
    // attention: consecutive query tiles per CTA (0 or 1: one)
    int q_per_cta;
    // bounded device waits give up after wait_ns (2 s unless a fault test shortens it)
    unsigned long long wait_ns;
    int dbg_skip_v;            // fault test only: the attention kernel's V producer issues nothing
};

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

__device__ __forceinline__ float sigmoidf_(float x) { return 1.0f / (1.0f + expf(-x)); }

}  // namespace hyb
