// token_level.cuh -- the token-level access variant of the inter-frame branch
// (fp32 CUDA-core kernels, any supported d).
//
// Source: "Technical summary: Attend Locally, Remember Linearly (ARL2)",
// gist.science/ar/paper/2605.16579, §4 (ablations: token-level against
// frame-level access to the memory).  The pages give no formulas; the reading
// (the library's API header states it too): on a clean pass the tokens of a
// frame update the state one after another by the frame-level rule applied to
// one token with a per-token forget gate,
//     S_t = alpha_t S_{t-1} + beta_t k'_t (v'_t - k'_t^T S_{t-1}),
//     alpha_t = sigmoid(g_t), beta_t = sigmoid(beta_logit_t),
// and token t reads the state before its own update, O_inter[t] = q'_t S_{t-1}.
//
// The recurrence is evaluated in chunks of kChunk tokens with only relative
// decays (Lambda_t = sum_{r<=t} log alpha_r within the chunk; every factor
// exp(Lambda_a - Lambda_b) has a >= b, so it lies in (0, 1] and nothing is
// divided by a gate).  Inside a chunk that starts from S, with u_t the row
// beta_t (v'_t - k'_t^T S_{t-1}):
//     (I + L) U = diag(beta) V' - diag(beta gprev) K' S,
//     L[t][s]   = beta_t exp(Lambda_{t-1} - Lambda_s) k'_t . k'_s   (s < t),
//     gprev_t   = exp(Lambda_{t-1}),
//     read_t    = gprev_t q'_t S + sum_{s<t} exp(Lambda_{t-1} - Lambda_s) (q'_t . k'_s) u_s,
//     S_end     = exp(Lambda_{C-1}) S + sum_s exp(Lambda_{C-1} - Lambda_s) k'_s u_s.
// Writing U = U0 - W S with [U0 | W] = (I + L)^{-1} [diag(beta) V' | diag(beta gprev) K']
// makes everything but a d x d chain independent of S:
//     S_end = M S + N,  M = exp(Lambda_{C-1}) I - K'^T diag(dec) W,  N = K'^T diag(dec) U0,
//     dec_s = exp(Lambda_{C-1} - Lambda_s).
// Three kernels, in stream order:
//   chunk_prep   (one block per chunk): projections, gates, L, the triangular
//                solve, M, N and the masked decayed Q'K'^T of the chunk;
//   chunk_chain  (one block per 16 state columns of a head): S_{c+1} = M_c S_c + N_c
//                over the chunks, saving every chunk's start state; writes S_N;
//   chunk_reads  (one block per chunk): the reads of the chunk's tokens, into an
//                fp32 buffer that the attention kernel adds to O_intra.
#pragma once

#include "common.cuh"
#include "sm100_ptx.cuh"

namespace hyb {
namespace tok {

constexpr int kChunk = 64;
constexpr int kThreads = 256;
constexpr int kBand = 16;  // state columns per chain block

// Per-(b, h, chunk) record in the workspace (floats), 256-byte aligned.
template <int D>
struct Rec {
    static constexpr size_t Qp = 0;                               // [C][D] q' = q phi_q^T
    static constexpr size_t Wm = Qp + (size_t)kChunk * D;         // [C][D] W
    static constexpr size_t U0 = Wm + (size_t)kChunk * D;         // [C][D] U0
    static constexpr size_t QK = U0 + (size_t)kChunk * D;         // [C][C] masked, decayed q'.k'
    static constexpr size_t GP = QK + (size_t)kChunk * kChunk;    // [C] gprev
    static constexpr size_t M = GP + kChunk;                      // [D][D] M^T (M[i][j] at j * D + i)
    static constexpr size_t N = M + (size_t)D * D;                // [D][D]
    static constexpr size_t S0 = N + (size_t)D * D;               // [D][D] the chunk's start state
    static constexpr size_t floats = (S0 + (size_t)D * D + 63) / 64 * 64;
};

template <int D>
struct PrepSmem {
    // phase 1: X [C][D+1] and phi^T [D][D]; K', V', Q' [C][D]; gates
    // phase 2 (reuses X / phi^T): L [C][C], [U0 | W] [C][2D]
    static constexpr size_t xs = (size_t)kChunk * (D + 1);
    static constexpr size_t ph = (size_t)D * (D + 1);   // phi^T, rows padded (no bank conflicts)
    static constexpr size_t region = (xs + ph) > ((size_t)kChunk * kChunk + (size_t)kChunk * 2 * D)
                                         ? (xs + ph)
                                         : ((size_t)kChunk * kChunk + (size_t)kChunk * 2 * D);
    static constexpr size_t bytes = sizeof(float) * (region + 3 * (size_t)kChunk * D + 4 * kChunk);
};

// Y[t][o] = sum_i X[t][i] phi[o][i] for the chunk's C rows (rows past T are 0).
template <int D, typename TIO>
__device__ __forceinline__ void project(const TIO* __restrict__ x, const TIO* __restrict__ phi, int t0, int T, int H,
                                        int h, int b, float* Xs, float* Ph, float* Y) {
    const int tid = threadIdx.x;
    for (int e = tid; e < kChunk * D; e += kThreads) {
        const int t = e / D, i = e % D;
        const int tok = t0 + t;
        Xs[t * (D + 1) + i] = tok < T ? to_f32(x[(((size_t)b * T + tok) * H + h) * D + i]) : 0.f;
    }
    const TIO* ph = phi + (size_t)h * D * D;
    for (int e = tid; e < D * D; e += kThreads) {
        const int o = e / D, i = e % D;
        Ph[i * (D + 1) + o] = to_f32(ph[e]);  // phi^T
    }
    __syncthreads();
    constexpr int CT = D / 16;           // columns per thread
    const int tg = tid / 16, og = tid % 16;
    float acc[4][CT];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < CT; ++c) acc[r][c] = 0.f;
    for (int i = 0; i < D; ++i) {
        float xr[4], pc[CT];
#pragma unroll
        for (int r = 0; r < 4; ++r) xr[r] = Xs[(tg * 4 + r) * (D + 1) + i];
#pragma unroll
        for (int c = 0; c < CT; ++c) pc[c] = Ph[i * (D + 1) + og + 16 * c];
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int c = 0; c < CT; ++c) acc[r][c] = fmaf(xr[r], pc[c], acc[r][c]);
    }
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < CT; ++c) Y[(tg * 4 + r) * D + og + 16 * c] = acc[r][c];
    __syncthreads();
}

template <int D, typename TIO>
__global__ void __launch_bounds__(kThreads) chunk_prep_kernel(LayerArgs a, float* __restrict__ rec_base) {
    using R = Rec<D>;
    using P = PrepSmem<D>;
    extern __shared__ float sm[];
    float* Xs = sm;                    // phase 1
    float* Ph = sm + P::xs;
    float* Ls = sm;                    // phase 2: [C][C]
    float* Sol = sm + (size_t)kChunk * kChunk;  // [C][2D]
    float* Kp = sm + P::region;        // [C][D]
    float* Vp = Kp + (size_t)kChunk * D;
    float* Qp = Vp + (size_t)kChunk * D;
    float* lam = Qp + (size_t)kChunk * D;   // Lambda_t
    float* bet = lam + kChunk;              // beta_t
    float* gpv = bet + kChunk;              // exp(Lambda_{t-1})
    float* dec = gpv + kChunk;              // exp(Lambda_{C-1} - Lambda_s)
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int T = a.T, H = a.H;
    const int t0 = c * kChunk;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t bh = (size_t)b * H + h;
    const int nch = (T + kChunk - 1) / kChunk;
    float* rec = rec_base + (bh * nch + c) * R::floats;

    // gates: beta_t and log alpha_t (0 for rows past T: they change nothing)
    if (warp == 0) {
        float la[2], be[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int t = lane + 32 * u, tok = t0 + t;
            const bool v = tok < T;
            const float g = v ? a.gate_logits[bh * T + tok] : 0.f;
            const float bl = v ? a.beta_logits[bh * T + tok] : 0.f;
            // log sigmoid(g) = -log(1 + exp(-g)), without overflow for large |g|
            la[u] = v ? (g >= 0.f ? -log1pf(expf(-g)) : g - log1pf(expf(g))) : 0.f;
            be[u] = v ? sigmoidf_(bl) : 0.f;
        }
        // inclusive prefix sum of log alpha over the 64 tokens
        float s0 = la[0], s1 = la[1];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y0 = __shfl_up_sync(0xffffffffu, s0, o), y1 = __shfl_up_sync(0xffffffffu, s1, o);
            if (lane >= o) {
                s0 += y0;
                s1 += y1;
            }
        }
        s1 += __shfl_sync(0xffffffffu, s0, 31);
        lam[lane] = s0;
        lam[lane + 32] = s1;
        bet[lane] = be[0];
        bet[lane + 32] = be[1];
    }
    __syncthreads();
    if (tid < kChunk) {
        const float lend = lam[kChunk - 1];
        gpv[tid] = tid == 0 ? 1.f : expf(lam[tid - 1]);
        dec[tid] = expf(fminf(lend - lam[tid], 0.f));
    }
    // projections
    project<D, TIO>((const TIO*)a.k, (const TIO*)a.phi_k, t0, T, H, h, b, Xs, Ph, Kp);
    project<D, TIO>((const TIO*)a.v, (const TIO*)a.phi_v, t0, T, H, h, b, Xs, Ph, Vp);
    project<D, TIO>((const TIO*)a.q, (const TIO*)a.phi_q, t0, T, H, h, b, Xs, Ph, Qp);
    // K' rows L2-normalised (a warp per row)
    for (int t = warp; t < kChunk; t += kThreads / 32) {
        float ss = 0.f;
        for (int i = lane; i < D; i += 32) ss = fmaf(Kp[t * D + i], Kp[t * D + i], ss);
        ss = warp_sum(ss);
        const float inv = t0 + t < T ? 1.0f / sqrtf(ss + a.l2_eps) : 0.f;
        for (int i = lane; i < D; i += 32) Kp[t * D + i] *= inv;
    }
    __syncthreads();
    // L (strictly lower, decayed, beta-scaled k'.k') and the masked decayed q'.k':
    // two 64 x 64 products over the features, from a transposed copy of K' (in
    // the projections' staging space, free now)
    {
        float* KT = sm + P::xs;  // [D][C]
        for (int e = tid; e < kChunk * D; e += kThreads) {
            const int t = e / D, i = e % D;
            KT[i * kChunk + t] = Kp[e];
        }
        __syncthreads();
        const int tg = tid / 16, sg = tid % 16;  // rows 4 tg..+3, columns sg + 16 c
        float dk[4][4], dq[4][4];
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int c = 0; c < 4; ++c) dk[r][c] = dq[r][c] = 0.f;
        for (int i = 0; i < D; ++i) {
            float kr[4], qr[4], ks[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                kr[r] = Kp[(tg * 4 + r) * D + i];
                qr[r] = Qp[(tg * 4 + r) * D + i];
            }
#pragma unroll
            for (int c = 0; c < 4; ++c) ks[c] = KT[i * kChunk + sg + 16 * c];
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    dk[r][c] = fmaf(kr[r], ks[c], dk[r][c]);
                    dq[r][c] = fmaf(qr[r], ks[c], dq[r][c]);
                }
        }
        __syncthreads();  // KT is overwritten by L below
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int t = tg * 4 + r, s2 = sg + 16 * c;
                float l = 0.f, qk = 0.f;
                if (s2 < t) {
                    const float dd = expf(fminf(lam[t - 1] - lam[s2], 0.f));
                    l = bet[t] * dd * dk[r][c];
                    qk = dd * dq[r][c];
                }
                Ls[t * kChunk + s2] = l;
                rec[R::QK + t * kChunk + s2] = qk;
            }
    }
    // right-hand sides [beta V' | beta gprev K'] and the forward substitution,
    // one column per thread
    for (int e = tid; e < kChunk * 2 * D; e += kThreads) {
        const int t = e / (2 * D), j = e % (2 * D);
        Sol[e] = j < D ? bet[t] * Vp[t * D + j] : bet[t] * gpv[t] * Kp[t * D + (j - D)];
    }
    __syncthreads();
    for (int j = tid; j < 2 * D; j += kThreads) {
        for (int t = 1; t < kChunk; ++t) {
            // four independent partial sums (the chain over s is the latency)
            float x0 = Sol[t * 2 * D + j], x1 = 0.f, x2 = 0.f, x3 = 0.f;
            int s = 0;
            for (; s + 4 <= t; s += 4) {
                x0 = fmaf(-Ls[t * kChunk + s], Sol[s * 2 * D + j], x0);
                x1 = fmaf(-Ls[t * kChunk + s + 1], Sol[(s + 1) * 2 * D + j], x1);
                x2 = fmaf(-Ls[t * kChunk + s + 2], Sol[(s + 2) * 2 * D + j], x2);
                x3 = fmaf(-Ls[t * kChunk + s + 3], Sol[(s + 3) * 2 * D + j], x3);
            }
            for (; s < t; ++s) x0 = fmaf(-Ls[t * kChunk + s], Sol[s * 2 * D + j], x0);
            Sol[t * 2 * D + j] = (x0 + x1) + (x2 + x3);
        }
    }
    __syncthreads();
    // U0, W, q', gprev for the reads
    for (int e = tid; e < kChunk * D; e += kThreads) {
        const int t = e / D, j = e % D;
        rec[R::U0 + e] = Sol[t * 2 * D + j];
        rec[R::Wm + e] = Sol[t * 2 * D + D + j];
        rec[R::Qp + e] = Qp[e];
    }
    if (tid < kChunk) rec[R::GP + tid] = gpv[tid];
    // M = exp(Lambda_{C-1}) I - K'^T diag(dec) W,  N = K'^T diag(dec) U0
    {
        const float gend = expf(lam[kChunk - 1]);
        constexpr int EI = D / 16;  // rows (and columns) per thread
        const int ig = tid / 16, jg = tid % 16;
        float m[EI][EI], nn[EI][EI];
#pragma unroll
        for (int p = 0; p < EI; ++p)
#pragma unroll
            for (int q = 0; q < EI; ++q) m[p][q] = nn[p][q] = 0.f;
        for (int s = 0; s < kChunk; ++s) {
            float kd[EI], w[EI], u[EI];
#pragma unroll
            for (int p = 0; p < EI; ++p) kd[p] = Kp[s * D + ig + 16 * p] * dec[s];
#pragma unroll
            for (int q = 0; q < EI; ++q) {
                w[q] = Sol[s * 2 * D + D + jg + 16 * q];
                u[q] = Sol[s * 2 * D + jg + 16 * q];
            }
#pragma unroll
            for (int p = 0; p < EI; ++p)
#pragma unroll
                for (int q = 0; q < EI; ++q) {
                    m[p][q] = fmaf(kd[p], w[q], m[p][q]);
                    nn[p][q] = fmaf(kd[p], u[q], nn[p][q]);
                }
        }
#pragma unroll
        for (int p = 0; p < EI; ++p)
#pragma unroll
            for (int q = 0; q < EI; ++q) {
                const int i = ig + 16 * p, j = jg + 16 * q;
                rec[R::M + (size_t)j * D + i] = (i == j ? gend : 0.f) - m[p][q];  // stored transposed
                rec[R::N + (size_t)i * D + j] = nn[p][q];
            }
    }
}

// S_{c+1} = M_c S_c + N_c over the chunks of one head, for kBand columns of S;
// every chunk's start state is saved for the reads, S_N goes to the state.
template <int D>
struct ChainSmem {
    // two M^T buffers (bulk copies, double-buffered), the band of S, two mbarriers
    static constexpr size_t bytes = sizeof(float) * (2 * (size_t)D * D + (size_t)D * kBand) + 64;
};

// S_{c+1} = M_c S_c + N_c over the chunks of one head, for kBand columns of S;
// every chunk's start state is saved for the reads, S_N goes to the state.
// M_{c+1}^T is copied into shared memory (one bulk copy) while step c runs.
template <int D>
__global__ void __launch_bounds__(D) chunk_chain_kernel(LayerArgs a, float* __restrict__ rec_base) {
    using R = Rec<D>;
    extern __shared__ __align__(128) float csm[];
    float* MT = csm;                                                  // [2][D][D]
    float (*Ss)[kBand] = reinterpret_cast<float (*)[kBand]>(csm + 2 * (size_t)D * D);
    uint64_t* bar = reinterpret_cast<uint64_t*>(csm + 2 * (size_t)D * D + (size_t)D * kBand);
    volatile int* abort_word = reinterpret_cast<volatile int*>(bar + 2);
    const int band = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int j0 = band * kBand;
    const int i = threadIdx.x;  // row of S
    const size_t bh = (size_t)b * a.H + h;
    const int nch = (a.T + kChunk - 1) / kChunk;
    float* S = a.state + bh * D * D;
    constexpr uint32_t kMBytes = (uint32_t)(D * D * sizeof(float));
    if (i == 0) {
        sm100::mbar_init(&bar[0], 1);
        sm100::mbar_init(&bar[1], 1);
        *abort_word = 0;
        sm100::fence_mbar_init();
        sm100::mbar_expect_tx(&bar[0], kMBytes);
        sm100::bulk_load(sm100::smem_u32(MT), rec_base + (bh * nch) * R::floats + R::M, kMBytes, &bar[0]);
    }
    __syncthreads();
    float s[kBand];
#pragma unroll
    for (int j = 0; j < kBand; ++j) s[j] = S[(size_t)i * D + j0 + j];
    bool ok = true;
    for (int c = 0; c < nch; ++c) {
        float* rec = rec_base + (bh * nch + c) * R::floats;
        const int buf = c & 1;
        if (i == 0 && c + 1 < nch) {
            // the other buffer was last read in step c - 1 (every thread passed the
            // barrier at its end): M_{c+1}^T goes there
            sm100::mbar_expect_tx(&bar[buf ^ 1], kMBytes);
            sm100::bulk_load(sm100::smem_u32(MT + (size_t)(buf ^ 1) * D * D), rec + R::floats + R::M, kMBytes,
                             &bar[buf ^ 1]);
        }
#pragma unroll
        for (int j = 0; j < kBand; ++j) {
            rec[R::S0 + (size_t)i * D + j0 + j] = s[j];
            Ss[i][j] = s[j];
        }
        float acc[kBand];
#pragma unroll
        for (int j = 0; j < kBand; ++j) acc[j] = rec[R::N + (size_t)i * D + j0 + j];
        ok = ok && sm100::mbar_wait(&bar[buf], (c >> 1) & 1, abort_word, a.flags, a.wait_ns);
        __syncthreads();
        if (ok) {
            const float* Mb = MT + (size_t)buf * D * D;
            for (int k = 0; k < D; ++k) {
                const float mik = Mb[k * D + i];
#pragma unroll
                for (int j = 0; j < kBand; ++j) acc[j] = fmaf(mik, Ss[k][j], acc[j]);
            }
        }
#pragma unroll
        for (int j = 0; j < kBand; ++j) s[j] = acc[j];
        __syncthreads();
    }
    bool bad = !ok;
#pragma unroll
    for (int j = 0; j < kBand; ++j) {
        S[(size_t)i * D + j0 + j] = s[j];
        bad |= !isfinite(s[j]);
    }
    if (__any_sync(0xffffffffu, bad) && (i & 31) == 0) atomicOr(a.flags, FLAG_NONFINITE);
}

template <int D>
struct ReadsSmem {
    static constexpr size_t bytes =
        sizeof(float) * ((size_t)D * D + 3 * (size_t)kChunk * D + (size_t)kChunk * kChunk + kChunk);
};

// read_t = gprev_t q'_t S_c + sum_s QK[t][s] (U0 - W S_c)[s], into out_tok [B][T][H][D]
template <int D>
__global__ void __launch_bounds__(kThreads) chunk_reads_kernel(LayerArgs a, const float* __restrict__ rec_base,
                                                               float* __restrict__ out_tok) {
    using R = Rec<D>;
    extern __shared__ float sm[];
    float* Sc = sm;                              // [D][D]
    float* Qs = Sc + (size_t)D * D;              // [C][D]
    float* Us = Qs + (size_t)kChunk * D;         // [C][D]: U0, then U0 - W S
    float* Ws = Us + (size_t)kChunk * D;         // [C][D]: W, then q' S
    float* QK = Ws + (size_t)kChunk * D;         // [C][C]
    float* gp = QK + (size_t)kChunk * kChunk;    // [C]
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int T = a.T;
    const int tid = threadIdx.x;
    const size_t bh = (size_t)b * a.H + h;
    const int nch = (T + kChunk - 1) / kChunk;
    const float* rec = rec_base + (bh * nch + c) * R::floats;
    for (int e = tid; e < D * D / 4; e += kThreads)
        reinterpret_cast<float4*>(Sc)[e] = reinterpret_cast<const float4*>(rec + R::S0)[e];
    for (int e = tid; e < kChunk * D / 4; e += kThreads) {
        reinterpret_cast<float4*>(Qs)[e] = reinterpret_cast<const float4*>(rec + R::Qp)[e];
        reinterpret_cast<float4*>(Us)[e] = reinterpret_cast<const float4*>(rec + R::U0)[e];
        reinterpret_cast<float4*>(Ws)[e] = reinterpret_cast<const float4*>(rec + R::Wm)[e];
    }
    for (int e = tid; e < kChunk * kChunk / 4; e += kThreads)
        reinterpret_cast<float4*>(QK)[e] = reinterpret_cast<const float4*>(rec + R::QK)[e];
    if (tid < kChunk) gp[tid] = rec[R::GP + tid];
    __syncthreads();
    constexpr int CT = D / 16;
    const int tg = tid / 16, og = tid % 16;  // rows 4 tg..+3, columns og + 16 c
    // W S and q' S for this thread's rows and columns
    float ws[4][CT], qs[4][CT];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int q = 0; q < CT; ++q) ws[r][q] = qs[r][q] = 0.f;
    for (int k = 0; k < D; ++k) {
        float sk[CT], wr[4], qr[4];
#pragma unroll
        for (int q = 0; q < CT; ++q) sk[q] = Sc[k * D + og + 16 * q];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            wr[r] = Ws[(tg * 4 + r) * D + k];
            qr[r] = Qs[(tg * 4 + r) * D + k];
        }
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int q = 0; q < CT; ++q) {
                ws[r][q] = fmaf(wr[r], sk[q], ws[r][q]);
                qs[r][q] = fmaf(qr[r], sk[q], qs[r][q]);
            }
    }
    __syncthreads();  // every thread has read W: reuse Ws for q' S
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int q = 0; q < CT; ++q) {
            const int t = tg * 4 + r, j = og + 16 * q;
            Us[t * D + j] -= ws[r][q];
            Ws[t * D + j] = gp[t] * qs[r][q];
        }
    __syncthreads();
    // + sum_s QK[t][s] U[s]
    float o[4][CT];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int q = 0; q < CT; ++q) o[r][q] = Ws[(tg * 4 + r) * D + og + 16 * q];
    for (int s = 0; s < kChunk; ++s) {
        float us[CT], qk[4];
#pragma unroll
        for (int q = 0; q < CT; ++q) us[q] = Us[s * D + og + 16 * q];
#pragma unroll
        for (int r = 0; r < 4; ++r) qk[r] = QK[(tg * 4 + r) * kChunk + s];
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int q = 0; q < CT; ++q) o[r][q] = fmaf(qk[r], us[q], o[r][q]);
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int tok = c * kChunk + tg * 4 + r;
        if (tok >= T) continue;
        float* dst = out_tok + (((size_t)b * T + tok) * a.H + h) * D;
#pragma unroll
        for (int q = 0; q < CT; ++q) dst[og + 16 * q] = o[r][q];
    }
}

}  // namespace tok
}  // namespace hyb
