// simt_layer.cuh -- fp32 CUDA-core (SIMT FFMA) kernels of the hybrid layer.
//
// Source: "Technical summary: Attend Locally, Remember Linearly (ARL2)",
// gist.science/ar/paper/2605.16579, §2.1 (intra-frame softmax branch,
// inter-frame read O_inter = Q' S_{N-1}, gated delta update) and §2.2
// (frame-level access, clean-pass updates).
//
// The pass is split into four kernels, in stream order:
//   prep       W = phi_q^T S_{N-1} per head (so that Q' S = Q W), and on a
//              clean pass a copy of S_{N-1} that the update reads;
//   attn       O_intra by online softmax over key tiles, plus O_inter = Q W,
//              written once as out = O_intra + O_inter;
//   partials   per token split: K' = rownorm(K phi_k^T), beta = sigmoid, and
//              the split's G = K'^T diag(beta) K' and P = K'^T diag(beta) V;
//   apply      S_N = alpha S_{N-1} + (sum P) phi_v^T - (sum G) S_{N-1}, with
//              alpha = mean_t sigmoid(g_t), summed over splits in fixed order.
// The last two are the delta rule regrouped:
//   K'^T diag(beta)(V phi_v^T - K' S) = (K'^T diag(beta) V) phi_v^T - (K'^T diag(beta) K') S.
#pragma once

#include "common.cuh"

namespace hyb {
namespace simt {

constexpr int kThreads = 256;

// ---------------------------------------------------------------- prep
// grid (D/R, H, B): block x computes rows k0..k0+R-1 of W = phi_q^T S (row-major
// fp32).  S and the block's R columns of phi_q are staged in shared memory; each
// warp owns R/8 rows of W and every lane D/32 consecutive columns.  (The
// tensor-core path computes W with tcgen05 in tc_kernels.cuh.)
constexpr int kRows = 16;
template <bool kSplitOut>
__host__ __device__ constexpr int prep_rows() { return 16; }

template <int D, int R>
struct PrepSmem {
    static constexpr size_t bytes = sizeof(float) * (D * D + D * R);
};

template <int D, typename TIO, bool kSplitOut>
__global__ void __launch_bounds__(kThreads) prep_kernel(LayerArgs a, int clean) {
    static_assert(!kSplitOut, "the bf16 hi + lo W is written by the tensor-core prep kernel");
    constexpr int NC = D / 32;
    constexpr int R = prep_rows<kSplitOut>();
    constexpr int RW = R / (kThreads / 32);  // rows of W per warp
    static_assert(RW == 2 || RW % 4 == 0, "rows per warp");
    extern __shared__ float smem[];
    float* Ss = smem;                  // [D][D]  S_{N-1}
    float* Ph = Ss + D * D;            // [D][R]  phi_q[o][k0 + kr]
    const int b = blockIdx.z, h = blockIdx.y, k0 = blockIdx.x * R;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t bh = (size_t)b * a.H + h;
    // all loads of a thread are issued before any shared-memory store: the
    // stores go through generic pointers, which would otherwise serialise them
    {
        const float4* S4 = reinterpret_cast<const float4*>(a.state + bh * D * D);
        constexpr int NS = D * D / 4 / kThreads;
        float4 sv[NS];
#pragma unroll
        for (int u = 0; u < NS; ++u) sv[u] = S4[tid + u * kThreads];
        const TIO* phiq = (const TIO*)a.phi_q + (size_t)h * D * D;
        constexpr int NP = D * R / kThreads;
        float pv[NP];
#pragma unroll
        for (int u = 0; u < NP; ++u) {
            const int i = tid + u * kThreads;
            pv[u] = to_f32(phiq[(i / R) * D + k0 + i % R]);
        }
#pragma unroll
        for (int u = 0; u < NS; ++u) reinterpret_cast<float4*>(Ss)[tid + u * kThreads] = sv[u];
#pragma unroll
        for (int u = 0; u < NP; ++u) Ph[tid + u * kThreads] = pv[u];
    }
    __syncthreads();
    // each warp owns rows r0..r0+RW-1 of W; each lane NC consecutive columns
    const int r0 = RW * warp;
    float acc[RW][NC];
#pragma unroll
    for (int q = 0; q < RW; ++q)
#pragma unroll
        for (int c = 0; c < NC; ++c) acc[q][c] = 0.f;
#pragma unroll 4
    for (int o = 0; o < D; ++o) {
        float p[RW];
        if constexpr (RW == 2) {
            const float2 p2 = *reinterpret_cast<const float2*>(Ph + o * R + r0);
            p[0] = p2.x;
            p[1] = p2.y;
        } else {
#pragma unroll
            for (int q = 0; q < RW; q += 4) {
                const float4 p4 = *reinterpret_cast<const float4*>(Ph + o * R + r0 + q);
                p[q] = p4.x;
                p[q + 1] = p4.y;
                p[q + 2] = p4.z;
                p[q + 3] = p4.w;
            }
        }
        float sv[NC];
#pragma unroll
        for (int c = 0; c < NC; ++c) sv[c] = Ss[o * D + NC * lane + c];
#pragma unroll
        for (int q = 0; q < RW; ++q)
#pragma unroll
            for (int c = 0; c < NC; ++c) acc[q][c] = fmaf(p[q], sv[c], acc[q][c]);
    }
    // branch combination: the inter-frame gain c folds into W (Q (c W) = c O_inter)
    if (a.mix) {
        const float cg = a.mix[bh * 2 + 1];
#pragma unroll
        for (int q = 0; q < RW; ++q)
#pragma unroll
            for (int c = 0; c < NC; ++c) acc[q][c] *= cg;
    }
#pragma unroll
    for (int rr = 0; rr < RW; ++rr) {
        const size_t row = bh * D * D + (size_t)(k0 + r0 + rr) * D + NC * lane;
#pragma unroll
        for (int c = 0; c < NC; ++c) a.W[row + c] = acc[rr][c];
    }
    if (clean) {
        // the fp32 update reads S_{N-1} from this copy (it writes the state in place)
        float4* dst = reinterpret_cast<float4*>(a.S_prev + bh * D * D + (size_t)k0 * D);
        for (int i = tid; i < R * D / 4; i += kThreads)
            dst[i] = reinterpret_cast<const float4*>(Ss + k0 * D)[i];
    }
}

// ---------------------------------------------------------------- attention
// grid (ceil(T/64), H, B); 8 warps x 8 query rows; lane j holds key j of a
// 32-key tile for the scores and columns lane + 32c of the outputs.
template <int D>
struct AttnSmem {
    static constexpr int BQ = 64, BK = 32;
    static constexpr size_t bytes = sizeof(float) * (BQ * D + BK * (D + 1) + BK * D);
};

template <int D, typename TIO>
__global__ void __launch_bounds__(kThreads) attn_kernel(LayerArgs a) {
    constexpr int BQ = AttnSmem<D>::BQ, BK = AttnSmem<D>::BK, NC = D / 32;
    extern __shared__ float smem[];
    float* Qs = smem;                  // [BQ][D]
    float* Ks = Qs + BQ * D;           // [BK][D+1]
    float* Vs = Ks + BK * (D + 1);     // [BK][D]
    const int b = blockIdx.z, h = blockIdx.y, q0 = blockIdx.x * BQ;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int T = a.T;
    const size_t rs = (size_t)a.H * D;  // elements between consecutive tokens
    const size_t base = (size_t)b * T * rs + (size_t)h * D;
    const TIO* q = (const TIO*)a.q + base;
    const TIO* k = (const TIO*)a.k + base;
    const TIO* v = (const TIO*)a.v + base;

    for (int i = tid; i < BQ * D; i += kThreads) {
        const int r = i / D, c = i % D, t = q0 + r;
        Qs[i] = t < T ? to_f32(q[(size_t)t * rs + c]) : 0.f;
    }
    float m[8], l[8], o[8][NC];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        m[r] = -INFINITY;
        l[r] = 0.f;
#pragma unroll
        for (int c = 0; c < NC; ++c) o[r][c] = 0.f;
    }
    const float* qrow = Qs + warp * 8 * D;
    for (int k0 = 0; k0 < T; k0 += BK) {
        __syncthreads();
        for (int i = tid; i < BK * D; i += kThreads) {
            const int r = i / D, c = i % D, t = k0 + r;
            Ks[r * (D + 1) + c] = t < T ? to_f32(k[(size_t)t * rs + c]) : 0.f;
            Vs[r * D + c] = t < T ? to_f32(v[(size_t)t * rs + c]) : 0.f;
        }
        __syncthreads();
        float s[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) s[r] = 0.f;
        for (int c = 0; c < D; ++c) {
            const float kc = Ks[lane * (D + 1) + c];
#pragma unroll
            for (int r = 0; r < 8; ++r) s[r] = fmaf(qrow[r * D + c], kc, s[r]);
        }
        const bool valid = (k0 + lane) < T;
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            const float sr = valid ? s[r] * a.sm_scale_log2 : -INFINITY;
            const float mnew = fmaxf(m[r], warp_max(sr));
            const float corr = exp2f(m[r] - mnew);
            const float p = exp2f(sr - mnew);
            l[r] = l[r] * corr + warp_sum(p);
            m[r] = mnew;
#pragma unroll
            for (int c = 0; c < NC; ++c) o[r][c] *= corr;
            s[r] = p;
        }
        for (int j = 0; j < BK; ++j) {
            float vj[NC];
#pragma unroll
            for (int c = 0; c < NC; ++c) vj[c] = Vs[j * D + lane + 32 * c];
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const float pj = __shfl_sync(0xffffffffu, s[r], j);
#pragma unroll
                for (int c = 0; c < NC; ++c) o[r][c] = fmaf(pj, vj[c], o[r][c]);
            }
        }
    }
    // inter-frame read: O_inter = Q (phi_q^T S)
    const float* W = a.W + ((size_t)b * a.H + h) * D * D;
    const float ag = a.mix ? a.mix[((size_t)b * a.H + h) * 2] : 1.0f;  // weight of O_intra in out
    float oe[8][NC];
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int c = 0; c < NC; ++c) oe[r][c] = 0.f;
    if (a.oi_ext) {
        // token-level access: the read was computed by the token-level kernels
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            const int t = q0 + warp * 8 + r;
            if (t >= T) continue;
            const float* src = a.oi_ext + (((size_t)b * T + t) * a.H + h) * D;
#pragma unroll
            for (int c = 0; c < NC; ++c) oe[r][c] = src[lane + 32 * c];
        }
    } else {
        for (int kk = 0; kk < D; ++kk) {
            float w[NC];
#pragma unroll
            for (int c = 0; c < NC; ++c) w[c] = W[kk * D + lane + 32 * c];
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const float qv = qrow[r * D + kk];
#pragma unroll
                for (int c = 0; c < NC; ++c) oe[r][c] = fmaf(qv, w[c], oe[r][c]);
            }
        }
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        const int t = q0 + warp * 8 + r;
        if (t >= T) continue;
        const float inv_l = 1.0f / l[r];
        const size_t row = (((size_t)b * T + t) * a.H + h) * D;
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            const int col = lane + 32 * c;
            const float intra = o[r][c] * inv_l;
            const float inter = oe[r][c];
            if (a.out) ((TIO*)a.out)[row + col] = from_f32<TIO>(fmaf(ag, intra, inter));
            if (a.out_intra) a.out_intra[row + col] = intra;
            if (a.out_inter) a.out_inter[row + col] = inter;
        }
    }
}

// ---------------------------------------------------------------- update partials
// grid (nsplit, H, B).  Per 32-token group: K' and beta*K' into shared memory,
// then every thread accumulates a (D/16) x (D/16) block of G and of P.
template <int D>
struct PartialsSmem {
    static constexpr size_t bytes =
        sizeof(float) * (D * (D + 1) + 32 * (D + 1) + 3 * 32 * D + 32);
};

template <int D, typename TIO>
__global__ void __launch_bounds__(kThreads, 1) partials_kernel(LayerArgs a) {
    constexpr int RI = D / 16, CJ = D / 16, NO = D / 8;
    extern __shared__ float smem[];
    float* phik = smem;                    // [D][D+1]
    float* Kr = phik + D * (D + 1);        // [32][D+1]
    float* Vr = Kr + 32 * (D + 1);         // [32][D]
    float* KU = Vr + 32 * D;               // [32][D]  K'
    float* Ab = KU + 32 * D;               // [32][D]  beta * K'
    float* betas = Ab + 32 * D;            // [32]
    const int b = blockIdx.z, h = blockIdx.y, split = blockIdx.x;
    const int tid = threadIdx.x;
    const int T = a.T;
    const size_t bh = (size_t)b * a.H + h;
    const size_t rs = (size_t)a.H * D;
    const size_t base = (size_t)b * T * rs + (size_t)h * D;
    const TIO* k = (const TIO*)a.k + base;
    const TIO* v = (const TIO*)a.v + base;
    const TIO* pk = (const TIO*)a.phi_k + (size_t)h * D * D;
    for (int i = tid; i < D * D; i += kThreads) phik[(i / D) * (D + 1) + i % D] = to_f32(pk[i]);

    const int t_begin = split * a.split_tokens;
    const int t_end = min(T, t_begin + a.split_tokens);
    const int ti = tid / 16, tj = tid % 16;
    float G[RI][CJ], P[RI][CJ];
#pragma unroll
    for (int r = 0; r < RI; ++r)
#pragma unroll
        for (int c = 0; c < CJ; ++c) G[r][c] = P[r][c] = 0.f;

    for (int t0 = t_begin; t0 < t_end; t0 += 32) {
        __syncthreads();
        for (int i = tid; i < 32 * D; i += kThreads) {
            const int r = i / D, c = i % D, t = t0 + r;
            Kr[r * (D + 1) + c] = t < t_end ? to_f32(k[(size_t)t * rs + c]) : 0.f;
            Vr[r * D + c] = t < t_end ? to_f32(v[(size_t)t * rs + c]) : 0.f;
        }
        if (tid < 32) {
            const int t = t0 + tid;
            betas[tid] = t < t_end ? sigmoidf_(a.beta_logits[bh * T + t]) : 0.f;
        }
        __syncthreads();
        {   // K~ = K phi_k^T for token tt, outputs o = og + 8j; then normalise
            const int tt = tid / 8, og = tid % 8;
            float kt[NO];
            float ss = 0.f;
#pragma unroll
            for (int j = 0; j < NO; ++j) {
                const float* prow = phik + (og + 8 * j) * (D + 1);
                const float* krow = Kr + tt * (D + 1);
                float acc = 0.f;
                for (int i = 0; i < D; ++i) acc = fmaf(prow[i], krow[i], acc);
                kt[j] = acc;
                ss = fmaf(acc, acc, ss);
            }
            ss += __shfl_xor_sync(0xffffffffu, ss, 1);
            ss += __shfl_xor_sync(0xffffffffu, ss, 2);
            ss += __shfl_xor_sync(0xffffffffu, ss, 4);
            const bool valid = (t0 + tt) < t_end;
            const float inv = valid ? 1.0f / sqrtf(ss + a.l2_eps) : 0.f;
            const float bt = betas[tt];
#pragma unroll
            for (int j = 0; j < NO; ++j) {
                const float ku = kt[j] * inv;
                KU[tt * D + og + 8 * j] = ku;
                Ab[tt * D + og + 8 * j] = ku * bt;
            }
        }
        __syncthreads();
        for (int tt = 0; tt < 32; ++tt) {
            float ai[RI], kj[CJ], vj[CJ];
#pragma unroll
            for (int r = 0; r < RI; ++r) ai[r] = Ab[tt * D + ti * RI + r];
#pragma unroll
            for (int c = 0; c < CJ; ++c) {
                kj[c] = KU[tt * D + tj + 16 * c];
                vj[c] = Vr[tt * D + tj + 16 * c];
            }
#pragma unroll
            for (int r = 0; r < RI; ++r)
#pragma unroll
                for (int c = 0; c < CJ; ++c) {
                    G[r][c] = fmaf(ai[r], kj[c], G[r][c]);
                    P[r][c] = fmaf(ai[r], vj[c], P[r][c]);
                }
        }
    }
    float* dst = a.partials + (bh * a.nsplit + split) * (size_t)D * 2 * D;
#pragma unroll
    for (int r = 0; r < RI; ++r)
#pragma unroll
        for (int c = 0; c < CJ; ++c) {
            const int i = ti * RI + r, j = tj + 16 * c;
            dst[(size_t)i * 2 * D + j] = G[r][c];
            dst[(size_t)i * 2 * D + D + j] = P[r][c];
        }
}

// ---------------------------------------------------------------- update apply
// grid (D/16, H, B): block x updates rows i0..i0+15 of S.  S_{N-1}, phi_v^T and
// the block's rows of sum G and sum P are staged in shared memory; each warp
// owns two rows, every lane the columns lane + 32c.
template <int D, typename TIO>
struct ApplySmem {
    static constexpr size_t bytes = sizeof(float) * (D * D + kRows * 2 * D + kThreads) +
                                    sizeof(TIO) * D * (D + 2);
};

template <int D, typename TIO>
__global__ void __launch_bounds__(kThreads) apply_kernel(LayerArgs a) {
    constexpr int NC = D / 32;
    extern __shared__ float smem[];
    float* Ss = smem;                          // [D][D]       S_{N-1}
    float* GP = Ss + D * D;                    // [16][2D]     rows of sum G | sum P
    float* red = GP + kRows * 2 * D;           // [kThreads]
    TIO* PvT = (TIO*)(red + kThreads);         // [D][D+2]     PvT[o][j] = phi_v[j][o]
    const int b = blockIdx.z, h = blockIdx.y, i0 = blockIdx.x * kRows;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int T = a.T;
    const size_t bh = (size_t)b * a.H + h;

    float sg = 0.f;
    for (int t = tid; t < T; t += kThreads) sg += sigmoidf_(a.gate_logits[bh * T + t]);
    red[tid] = sg;
    const float4* S4 = reinterpret_cast<const float4*>(a.S_prev + bh * D * D);
    for (int i = tid; i < D * D / 4; i += kThreads) reinterpret_cast<float4*>(Ss)[i] = S4[i];
    const TIO* pv = (const TIO*)a.phi_v + (size_t)h * D * D;
    for (int i = tid; i < D * D; i += kThreads) PvT[(i % D) * (D + 2) + i / D] = pv[i];
    {   // fixed-order sum over the token splits; all loads of a split in flight together
        constexpr int PER = kRows * 2 * D / kThreads;
        float acc[PER];
#pragma unroll
        for (int q = 0; q < PER; ++q) acc[q] = 0.f;
        const float* base = a.partials + (bh * a.nsplit * D + i0) * (size_t)2 * D;
        for (int sp = 0; sp < a.nsplit; ++sp) {
            const float* src = base + (size_t)sp * D * 2 * D;
#pragma unroll
            for (int q = 0; q < PER; ++q) acc[q] += src[tid + q * kThreads];
        }
#pragma unroll
        for (int q = 0; q < PER; ++q) GP[tid + q * kThreads] = acc[q];
    }
    __syncthreads();
    for (int st = kThreads / 2; st > 0; st >>= 1) {
        if (tid < st) red[tid] += red[tid + st];
        __syncthreads();
    }
    const float alpha = red[0] / (float)T;

    const int r0 = 2 * warp;
    float acc[2][NC];
#pragma unroll
    for (int rr = 0; rr < 2; ++rr)
#pragma unroll
        for (int c = 0; c < NC; ++c) acc[rr][c] = alpha * Ss[(i0 + r0 + rr) * D + lane + 32 * c];
    const float* G0 = GP + r0 * 2 * D;
    const float* G1 = G0 + 2 * D;
#pragma unroll 4
    for (int o = 0; o < D; ++o) {
        const float p0 = G0[D + o], p1 = G1[D + o];
        const float g0 = G0[o], g1 = G1[o];
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            const int j = lane + 32 * c;
            const float f = to_f32(PvT[o * (D + 2) + j]);
            const float sv = Ss[o * D + j];
            acc[0][c] = fmaf(p0, f, acc[0][c]);
            acc[1][c] = fmaf(p1, f, acc[1][c]);
            acc[0][c] = fmaf(-g0, sv, acc[0][c]);
            acc[1][c] = fmaf(-g1, sv, acc[1][c]);
        }
    }
    bool bad = false;
    float* S = a.state + bh * D * D;
#pragma unroll
    for (int rr = 0; rr < 2; ++rr)
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            S[(size_t)(i0 + r0 + rr) * D + lane + 32 * c] = acc[rr][c];
            bad |= !isfinite(acc[rr][c]);
        }
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(a.flags, FLAG_NONFINITE);
}

}  // namespace simt
}  // namespace hyb
