// tc_kernels.cuh -- tensor-core (tcgen05 / TMEM / TMA) delta update of the
// hybrid layer for bf16 I/O and d = 128 on sm_100a.
//
// Source: "Technical summary: Attend Locally, Remember Linearly (ARL2)",
// gist.science/ar/paper/2605.16579, §2.1 (intra-frame softmax branch,
// inter-frame read O_inter = Q' S_{N-1}, gated delta update) and §2.2
// (frame-level access: all tokens read the pre-update state).
//
// The attention kernel is in tc_attention.cuh; this file holds the operand
// descriptors both use and the delta update.
//
// delta_update: one cluster per (head, batch), one CTA per token split.  Per
// 128-token tile: K~ = K phi_k^T on the tensor core, row L2-normalisation and
// beta in registers, then G += (beta K')^T K' and P += (beta K')^T V as
// MN-major contractions over the tokens, with beta K' and K' split into bf16
// hi + lo (G takes hi*hi + hi*lo + lo*hi, P takes hi*V + lo*V; V is exact in
// bf16); the splits are then reduced through distributed shared memory and
// the update is applied in fp32 (see the kernel's comment).
#pragma once

#include "common.cuh"
#include "sm100_ptx.cuh"

namespace hyb {
namespace tc {

using namespace sm100;

constexpr int kTile = 128;
constexpr uint32_t kTileBytes = 128 * 128 * 2;  // one 128 x 128 bf16 tile
constexpr uint32_t kHalf = kTileBytes / 2;      // one 128 x 64 TMA box
constexpr int kMaxClusterRanks = 8;             // token splits per (b, h) in the update


// K-major operand, 128 rows x 128 bf16 stored as two 64-column swizzled boxes:
// descriptor of the 16-column slice kk (0..7).
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t base, int kk) {
    return sdesc_sw128(base + (kk >> 2) * kHalf + (kk & 3) * 32, 16, 1024);
}
// MN-major operand with the same storage (rows = K index): slice kk covers K rows 16kk..16kk+15.
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t base, int kk) {
    return sdesc_sw128(base + kk * 2048, kHalf, 1024);
}

// A descriptor's start-address field is its low 14 bits (the shared-memory
// address / 16, all addresses below 256 KB), so the descriptor of slice kk is
// the tile's descriptor (slice 0) plus a constant; the MMA issuing thread then
// spends one add per MMA on its operands.
__device__ __forceinline__ uint64_t kmajor_step(int kk) { return (uint64_t)((kk >> 2) * (kHalf >> 4) + (kk & 3) * 2); }
__device__ __forceinline__ uint64_t mnmajor_step(int kk) { return (uint64_t)(kk * (2048 >> 4)); }

// Eight MMAs D (+)= A_kk B_kk over the K slices kk = 0..7 of one 128-deep
// product, A in TMEM (columns a_tmem + 8 kk), B from shared-memory descriptors
// b0 + step(kk); the first accumulates into D if acc0, the rest always.
template <bool kMnB>
__device__ __forceinline__ void mma8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b0, uint32_t idesc, uint32_t acc0) {
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
        mma_bf16_ts(d_tmem, a_tmem + kk * 8, b0 + (kMnB ? mnmajor_step(kk) : kmajor_step(kk)), idesc,
                    kk > 0 ? 1u : acc0);
}

// The same with A from shared memory too: a K-major tile with descriptor a0 + step(kk).
template <bool kMnB>
__device__ __forceinline__ void mma8_ss(uint32_t d_tmem, uint64_t a0, uint64_t b0, uint32_t idesc, uint32_t acc0) {
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
        mma_bf16(d_tmem, a0 + kmajor_step(kk), b0 + (kMnB ? mnmajor_step(kk) : kmajor_step(kk)), idesc,
                 kk > 0 ? 1u : acc0);
}

// Max of N scores (fmaxf: NaN entries are skipped).
template <int N>
__device__ __forceinline__ float row_max(const float* x) {
    float m8[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) m8[k] = x[k];
#pragma unroll
    for (int c = 8; c < N; ++c) m8[c & 7] = fmaxf(m8[c & 7], x[c]);
    return fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
}

// ============================================================== delta update
// One cluster of C CTAs per (batch, head); CTA c of the cluster takes token
// split c (a run of 128-token tiles) and accumulates its G_c = (beta K')^T K'
// and P_c = (beta K')^T V in TMEM.  Since the update is linear in the splits,
// every CTA then forms its own contribution Delta_c = P_c phi_v^T - G_c S_{N-1}
// on the tensor core (bf16 hi + lo splits of G_c, P_c and S_{N-1}), and each
// CTA sums one band of rows of Delta over the C CTAs through distributed
// shared memory (fixed order c = 0..C-1, so the result is deterministic):
//   S_N[i][:] = alpha S_{N-1}[i][:] + sum_c Delta_c[i][:]
// with alpha = mean_t sigmoid(g_t).  Every CTA stages S_{N-1} from the state
// buffer before the cluster's first barrier and writes its band after it.  The
// kernel reads only the pass's inputs and the state, never the prep kernel's
// outputs, so it may run alongside the attention kernel.
namespace upd {
// tile loop (1024-aligned 128B-swizzled tiles)
constexpr uint32_t PHI = 0;
constexpr uint32_t KT = PHI + kTileBytes;
constexpr uint32_t VT = KT + kTileBytes;
constexpr uint32_t AH = VT + kTileBytes;
constexpr uint32_t AL = AH + kTileBytes;
constexpr uint32_t KH = AL + kTileBytes;
constexpr uint32_t KL = KH + kTileBytes;
constexpr uint32_t TILES_END = KL + kTileBytes;          // 229,376
// after the tile loop (reuses the tile space)
constexpr uint32_t PHIV = 0;                              // phi_v, K-major B operand (rows j, o contiguous)
constexpr uint32_t SPREV = PHIV + kTileBytes;             // S_{N-1} fp32 [128][128]
constexpr uint32_t SH = SPREV + 128 * 128 * 4;            // S_hi, MN-major B operand (rows m, j contiguous)
constexpr uint32_t SL = SH + kTileBytes;                  // S_lo
constexpr uint32_t RED = SL + kTileBytes;                 // Delta_c fp32 [128][128], 16-byte chunks XOR-swizzled
constexpr uint32_t BAR = TILES_END;                       // barriers, TMEM slot, flags, sums
constexpr uint32_t XSS = BAR + 256;                       // [2 parity][2 halves][128 rows] floats + ok bytes
constexpr uint32_t SMEM = XSS + 2048 + 512;               // 232,192 B
constexpr int kNormThreads = 256;                         // warps 0-7
constexpr int kLoadWarp = 8, kMmaWarp = 9;
constexpr int kThreads = 320;
enum { B_PHI = 0, B_KFULL, B_KFREE, B_VFULL, B_KTFULL, B_KTFULL1, B_KTREAD, B_KTREAD1, B_OPSFULL, B_OPSFREE,
       B_PARK, B_DELTA, B_WPHI, B_WMMA, B_DRAIN, B_COUNT };
static_assert(RED + 128 * 128 * 4 <= TILES_END, "post-loop buffers exceed the tile space");
// byte offset of float4 chunk q (0..31) of row `row` in RED
__device__ __forceinline__ uint32_t red_off(int row, int q) {
    return (uint32_t)(row * 512 + ((q ^ (row & 7)) << 4));
}
}  // namespace upd

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_nctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ float4 ld_cluster_f4(uint32_t local_addr, uint32_t rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_addr), "r"(rank));
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(remote)
                 : "memory");
    return v;
}

__global__ void __launch_bounds__(upd::kThreads, 1)
    update_kernel(const __grid_constant__ LayerArgs a, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_phik,
                  const __grid_constant__ CUtensorMap tm_phiq) {
    using namespace upd;
    extern __shared__ __align__(1024) uint8_t smem[];
    if (smem_u32(smem) & 1023u) {  // uniform over the grid: every CTA leaves
        if (threadIdx.x == 0) atomicOr(a.flags, FLAG_INTERNAL);
        return;
    }
    // a chained pass: the next kernel of the stream (the next pass's attention,
    // which reads W of the next frame only after this grid completes) may start
    // on the SMs this grid leaves idle
    if (a.chain_trigger == 1) pdl_launch_dependents();
    const uint32_t sb = smem_u32(smem);
    uint64_t* bars = (uint64_t*)(smem + BAR);
    uint32_t* tmem_slot = (uint32_t*)(bars + B_COUNT);
    volatile int* abort_word = (volatile int*)(tmem_slot + 1);
    float* wsum = (float*)(tmem_slot + 2);  // 10 warp partial sums + alpha
    float* xss = (float*)(smem + XSS);      // row sums of squares exchanged between warp pairs
    uint8_t* xok = smem + XSS + 2048;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.y, b = blockIdx.z;
    const int split = (int)cluster_ctarank();
    const int C = (int)cluster_nctarank();
    const int T = a.T;
    const int bh = b * a.H + h;
    const int t_begin = split * a.split_tokens;
    const int t_end = min(T, t_begin + a.split_tokens);
    const int nt = t_end > t_begin ? (t_end - t_begin + kTile - 1) / kTile : 0;
    // this thread's first gate logits (for alpha), loaded now and summed after the tile loop
    const float* gl = a.gate_logits + (size_t)bh * T;
    float g0[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) g0[u] = (threadIdx.x + u * kThreads < T) ? gl[threadIdx.x + u * kThreads] : 0.f;

    if (threadIdx.x == 0) {
        for (int i = 0; i < B_COUNT; ++i)
            mbar_init(&bars[i], (i == B_OPSFULL || i == B_KTREAD || i == B_KTREAD1) ? kNormThreads : 1);
        *abort_word = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) tmem_alloc(tmem_slot, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // K~ of tile i in buffer i & 1 (columns [0,128) or [384,512)), so the K phi_k^T
    // product of the next tile runs while this one is normalised
    const uint32_t tG = tmem + 128, tP = tmem + 256;
    auto tKT = [&](int i) { return (i & 1) ? tmem + 384 : tmem; };

    uint4 pv[8];  // phi_v staging (normalisation warps)
    // ------------------------------------------------------------ tile loop
    if (warp == kLoadWarp) {
        if (lane == 0 && nt > 0) {
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            tma_prefetch_desc(&tm_phik);
            const int xh = h * 128;
            mbar_expect_tx(&bars[B_PHI], kTileBytes);
            tma_load_3d(sb + PHI, &tm_phik, &bars[B_PHI], 0, 0, h);
            tma_load_3d(sb + PHI + kHalf, &tm_phik, &bars[B_PHI], 64, 0, h);
            for (int i = 0; i < nt; ++i) {
                const int t0 = t_begin + i * kTile;
                if (i > 0 && !mbar_wait(&bars[B_KFREE], (i - 1) & 1, abort_word, a.flags)) break;
                mbar_expect_tx(&bars[B_KFULL], kTileBytes);
                tma_load_3d(sb + KT, &tm_k, &bars[B_KFULL], xh, t0, b);
                tma_load_3d(sb + KT + kHalf, &tm_k, &bars[B_KFULL], xh + 64, t0, b);
                if (i > 0 && !mbar_wait(&bars[B_OPSFREE], (i - 1) & 1, abort_word, a.flags)) break;
                mbar_expect_tx(&bars[B_VFULL], kTileBytes);
                tma_load_3d(sb + VT, &tm_v, &bars[B_VFULL], xh, t0, b);
                tma_load_3d(sb + VT + kHalf, &tm_v, &bars[B_VFULL], xh + 64, t0, b);
            }
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        if (lane == 0 && nt > 0) {
            constexpr uint32_t ID_KK = idesc_bf16(128, 128, 0, 0);
            constexpr uint32_t ID_MNMN = idesc_bf16(128, 128, 1, 1);
            // K~(i+1) = K_{i+1} phi_k^T is issued ahead of tile i's G and P products,
            // so the next tile's normalisation can start while they run
            bool ok = mbar_wait(&bars[B_PHI], 0, abort_word, a.flags) &&
                      mbar_wait(&bars[B_KFULL], 0, abort_word, a.flags);
            if (ok) {
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16(tKT(0), kmajor_desc(sb + KT, kk), kmajor_desc(sb + PHI, kk), ID_KK, kk > 0);
                mma_commit(&bars[B_KTFULL]);
                mma_commit(&bars[B_KFREE]);
            }
            for (int i = 0; i < nt && ok; ++i) {
                if (i + 1 < nt) {
                    if (!(ok = mbar_wait(&bars[B_KFULL], (i + 1) & 1, abort_word, a.flags))) break;
                    // the buffer of K~(i+1) was last read by the normalisation of tile i-1
                    if (i >= 1 && !(ok = mbar_wait(&bars[B_KTREAD + ((i + 1) & 1)], ((i - 1) >> 1) & 1,
                                                   abort_word, a.flags)))
                        break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_bf16(tKT(i + 1), kmajor_desc(sb + KT, kk), kmajor_desc(sb + PHI, kk), ID_KK, kk > 0);
                    mma_commit(&bars[B_KTFULL + ((i + 1) & 1)]);
                    mma_commit(&bars[B_KFREE]);
                }
                if (!(ok = mbar_wait(&bars[B_OPSFULL], i & 1, abort_word, a.flags))) break;
                tc_fence_after();
                // G first: it does not need this tile's V, whose load starts only
                // once the previous tile's P products have read the V buffer
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t acc = (i > 0 || kk > 0);
                    mma_bf16(tG, mnmajor_desc(sb + AH, kk), mnmajor_desc(sb + KH, kk), ID_MNMN, acc);
                    mma_bf16(tG, mnmajor_desc(sb + AH, kk), mnmajor_desc(sb + KL, kk), ID_MNMN, 1);
                    mma_bf16(tG, mnmajor_desc(sb + AL, kk), mnmajor_desc(sb + KH, kk), ID_MNMN, 1);
                }
                if (!(ok = mbar_wait(&bars[B_VFULL], i & 1, abort_word, a.flags))) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t acc = (i > 0 || kk > 0);
                    mma_bf16(tP, mnmajor_desc(sb + AH, kk), mnmajor_desc(sb + VT, kk), ID_MNMN, acc);
                    mma_bf16(tP, mnmajor_desc(sb + AL, kk), mnmajor_desc(sb + VT, kk), ID_MNMN, 1);
                }
                mma_commit(&bars[B_OPSFREE]);
            }
            // drain: every MMA issued so far completes before the tile space is reused
            mma_commit(&bars[B_PHI]);
            uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(smem_u32(&bars[B_PHI]), 1) && globaltimer_ns() - t0 < kWaitNs) {
            }
        }
        __syncwarp();
    } else {
        // Warps w and w+4 share token rows (TMEM lanes 32(w%4)..+31); warp w/4 = half
        // takes feature columns 64*half..64*half+63.  The pair exchanges its half
        // sums of squares (and wait results) at a named barrier every tile.
        const int half = warp >> 2;
        const int r = (warp & 3) * 32 + lane;
        const int pair_bar = 1 + (warp & 3);
        const uint32_t lrow = (uint32_t)((warp & 3) * 32) << 16;
        bool ok = true;
        float x[64];
        for (int i = 0; i < nt; ++i) {
            const int s = i & 1;
            // this row's beta logit, loaded before the wait for K~
            const int tok = t_begin + i * kTile + r;
            const bool valid = tok < t_end;
            const float bl = valid ? a.beta_logits[(size_t)bh * T + tok] : 0.f;
            bool w_ok = __all_sync(0xffffffffu,
                                   ok && mbar_wait(&bars[B_KTFULL + (i & 1)], (i >> 1) & 1, abort_word, a.flags));
            float ssh = 0.f;
            if (w_ok) {
                tc_fence_after();
                tmem_ld32(tKT(i) + lrow + half * 64, x);
                tmem_ld32(tKT(i) + lrow + half * 64 + 32, x + 32);
                tmem_ld_wait();
                tc_fence_before();
                mbar_arrive(&bars[B_KTREAD + (i & 1)]);  // K~(i+2) may overwrite this buffer
                float ss8[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) ss8[k] = 0.f;
#pragma unroll
                for (int c = 0; c < 64; ++c) ss8[c & 7] = fmaf(x[c], x[c], ss8[c & 7]);
                ssh = ((ss8[0] + ss8[1]) + (ss8[2] + ss8[3])) + ((ss8[4] + ss8[5]) + (ss8[6] + ss8[7]));
            }
            xss[(s * 2 + half) * 128 + r] = ssh;
            xok[(s * 2 + half) * 128 + r] = (uint8_t)w_ok;
            named_bar_sync(pair_bar, 64);
            ok = __all_sync(0xffffffffu, w_ok && xok[(s * 2 + (half ^ 1)) * 128 + r]);
            if (!ok) continue;  // keep arriving at the pair barriers until the loop ends
            // the operand tiles are free once the previous tile's products have read them
            if (i > 0) ok = __all_sync(0xffffffffu, mbar_wait(&bars[B_OPSFREE], (i - 1) & 1, abort_word, a.flags));
            if (!ok) continue;
            const float ss = xss[(s * 2 + 0) * 128 + r] + xss[(s * 2 + 1) * 128 + r];
            const float inv = valid ? 1.0f / sqrtf(ss + a.l2_eps) : 0.f;
            const float beta = valid ? sigmoidf_(bl) : 0.f;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                uint32_t ah[4], al[4], kh[4], kl[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int col = c * 8 + 2 * q;
                    const float k0 = x[col] * inv, k1 = x[col + 1] * inv;
                    const float a0 = k0 * beta, a1 = k1 * beta;
                    const __nv_bfloat162 khv = __floats2bfloat162_rn(k0, k1);
                    const __nv_bfloat162 ahv = __floats2bfloat162_rn(a0, a1);
                    kh[q] = *reinterpret_cast<const uint32_t*>(&khv);
                    ah[q] = *reinterpret_cast<const uint32_t*>(&ahv);
                    kl[q] = pack_bf16(k0 - __low2float(khv), k1 - __high2float(khv));
                    al[q] = pack_bf16(a0 - __low2float(ahv), a1 - __high2float(ahv));
                }
                const uint32_t off = half * kHalf + sw128_offset(r, c);
                *reinterpret_cast<uint4*>(smem + AH + off) = make_uint4(ah[0], ah[1], ah[2], ah[3]);
                *reinterpret_cast<uint4*>(smem + AL + off) = make_uint4(al[0], al[1], al[2], al[3]);
                *reinterpret_cast<uint4*>(smem + KH + off) = make_uint4(kh[0], kh[1], kh[2], kh[3]);
                *reinterpret_cast<uint4*>(smem + KL + off) = make_uint4(kl[0], kl[1], kl[2], kl[3]);
            }
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(&bars[B_OPSFULL]);
        }
        // phi_v row r, columns 64 half..+63, loaded while the last products run
        {
            const uint4* src = reinterpret_cast<const uint4*>((const __nv_bfloat16*)a.phi_v +
                                                              (size_t)h * 128 * 128 + (size_t)r * 128 + half * 64);
#pragma unroll
            for (int c = 0; c < 8; ++c) pv[c] = src[c];
        }
        if (ok && nt > 0)
            ok = __all_sync(0xffffffffu, mbar_wait(&bars[B_OPSFREE], (nt - 1) & 1, abort_word, a.flags));
    }
    // ------------------------------------------------------------ Delta_c = P_c phi_v^T - G_c S_{N-1}
    // G_c and P_c (fp32 in TMEM) become bf16 hi + lo A operands in TMEM; S_{N-1}
    // becomes a bf16 hi + lo B operand and phi_v a K-major B operand in shared
    // memory; five MMAs give this split's contribution, which the cluster sums.
    const uint32_t tGH = tmem, tGL = tmem + 64, tD = tmem + 128, tPH = tmem + 384, tPL = tmem + 448;
    tc_fence_before();
    __syncthreads();  // every MMA of the tile loop has completed (or timed out)
    tc_fence_after();
    // the next update of a chain of updates (its key tiles need nothing from
    // this one) may start once every CTA here has finished its key tiles
    if (a.chain_trigger == 2) pdl_launch_dependents();
    bool park_issued = false, wphi_issued = false;  // (loader) copies to drain before exit
    if (threadIdx.x == kLoadWarp * 32) {
        // a chained pass may have started before the previous chained update has
        // written S_{N-1}: wait for its flags (every CTA of its cluster raises one
        // once it is done with the state), then read the state through the async proxy
        bool chain_ok = true;
        if (a.chain_wait) {
            chain_ok = flags_wait_equal(a.chain_flags + (size_t)bh * kMaxClusterRanks, C, a.chain_wait, a.flags,
                                        a.wait_ns);
            fence_proxy_async_all();
        }
        if (chain_ok) {
            mbar_expect_tx(&bars[B_PARK], 128 * 128 * 4);
            bulk_load(sb + SPREV, a.state + (size_t)bh * 128 * 128, 128 * 128 * 4, &bars[B_PARK]);
            park_issued = true;
        } else {
            *abort_word = 1;  // nothing in flight; every later wait of the CTA gives up
        }
    }
    {
        // alpha: the entry loads, then any further logits (T > 8 x 320), each
        // batch loaded before its sigmoids are taken
        float sg = 0.f;
#pragma unroll
        for (int u = 0; u < 8; ++u)
            if (threadIdx.x + u * kThreads < T) sg += sigmoidf_(g0[u]);
        for (int t0 = threadIdx.x + 8 * kThreads; t0 < T; t0 += 8 * kThreads) {
            float g[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) g[u] = (t0 + u * kThreads < T) ? gl[t0 + u * kThreads] : 0.f;
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (t0 + u * kThreads < T) sg += sigmoidf_(g[u]);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sg += __shfl_xor_sync(0xffffffffu, sg, o);
        if (lane == 0) wsum[warp] = sg;
    }
    bool park_ok = true;
    if (warp < 8) {
        const int half = warp >> 2;
        const int row = (warp & 3) * 32 + lane;
        const uint32_t lrow = (uint32_t)((warp & 3) * 32) << 16;
        // phi_v row `row`, columns 64 half..+63 (loaded during the tile loop), into the K-major B tile
#pragma unroll
        for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(smem + PHIV + half * kHalf + sw128_offset(row, c)) = pv[c];
        // G and P rows `row`, columns 64 half..+63: fp32 -> bf16 hi + lo in TMEM
#pragma unroll
        for (int gp = 0; gp < 2; ++gp) {
            float x[64];
            uint32_t hi[32], lo[32];
            const uint32_t src = (gp == 0 ? tG : tP) + lrow + half * 64;
            if (nt > 0) {
                tmem_ld32(src, x);
                tmem_ld32(src + 32, x + 32);
                tmem_ld_wait();
            } else {
#pragma unroll
                for (int q = 0; q < 64; ++q) x[q] = 0.f;
            }
#pragma unroll
            for (int q = 0; q < 32; ++q) {
                const __nv_bfloat162 hv = __floats2bfloat162_rn(x[2 * q], x[2 * q + 1]);
                hi[q] = *reinterpret_cast<const uint32_t*>(&hv);
                lo[q] = pack_bf16(x[2 * q] - __low2float(hv), x[2 * q + 1] - __high2float(hv));
            }
            tmem_st32u((gp == 0 ? tGH : tPH) + lrow + half * 32, hi);
            tmem_st32u((gp == 0 ? tGL : tPL) + lrow + half * 32, lo);
        }
        tmem_st_wait();
        // S_{N-1} row `row`, columns 64 half..+63: bf16 hi + lo into the MN-major B tiles
        park_ok = __all_sync(0xffffffffu, mbar_wait(&bars[B_PARK], 0, abort_word, a.flags));
        // float4 k of the row half is read in the order (k0 + lane) & 15, so a
        // warp's reads (rows 512 B apart) spread over all 16-byte bank groups
        const float4* Sp4 = reinterpret_cast<const float4*>(smem + SPREV) + row * 32 + half * 16;
#pragma unroll
        for (int k0 = 0; k0 < 16; ++k0) {
            const int k = (k0 + lane) & 15;
            const float4 v = Sp4[k];
            const __nv_bfloat162 h01 = __floats2bfloat162_rn(v.x, v.y);
            const __nv_bfloat162 h23 = __floats2bfloat162_rn(v.z, v.w);
            const uint2 hi = make_uint2(*reinterpret_cast<const uint32_t*>(&h01), *reinterpret_cast<const uint32_t*>(&h23));
            const uint2 lo = make_uint2(pack_bf16(v.x - __low2float(h01), v.y - __high2float(h01)),
                                        pack_bf16(v.z - __low2float(h23), v.w - __high2float(h23)));
            const uint32_t off = half * kHalf + sw128_offset(row, k >> 1) + (k & 1) * 8;
            *reinterpret_cast<uint2*>(smem + SH + off) = hi;
            *reinterpret_cast<uint2*>(smem + SL + off) = lo;
        }
    } else {
        // S_{N-1} must be in shared memory before any CTA of the cluster passes the
        // first cluster barrier: after it, CTAs write their bands of the state
        park_ok = __all_sync(0xffffffffu, mbar_wait(&bars[B_PARK], 0, abort_word, a.flags));
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (threadIdx.x == kMmaWarp * 32) {
        constexpr uint32_t ID_KK = idesc_bf16(128, 128, 0, 0);
        constexpr uint32_t ID_KMN_NEG = idesc_bf16(128, 128, 0, 1) | (1u << 13);  // -A
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) mma_bf16_ts(tD, tPH + kk * 8, kmajor_desc(sb + PHIV, kk), ID_KK, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) mma_bf16_ts(tD, tPL + kk * 8, kmajor_desc(sb + PHIV, kk), ID_KK, 1);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) mma_bf16_ts(tD, tGH + kk * 8, mnmajor_desc(sb + SH, kk), ID_KMN_NEG, 1);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) mma_bf16_ts(tD, tGH + kk * 8, mnmajor_desc(sb + SL, kk), ID_KMN_NEG, 1);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) mma_bf16_ts(tD, tGL + kk * 8, mnmajor_desc(sb + SH, kk), ID_KMN_NEG, 1);
        mma_commit(&bars[B_DELTA]);
    }
    if (warp < 8) {
        // Delta_c row `row`, columns 64 half..+63, into shared memory for the cluster
        const int half = warp >> 2;
        const int row = (warp & 3) * 32 + lane;
        const uint32_t lrow = (uint32_t)((warp & 3) * 32) << 16;
        const bool d_ok = __all_sync(0xffffffffu, mbar_wait(&bars[B_DELTA], 0, abort_word, a.flags));
        tc_fence_after();
        float v[32];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            if (d_ok) {
                tmem_ld32(tD + lrow + half * 64 + c * 32, v);
                tmem_ld_wait();
            } else {
#pragma unroll
                for (int q = 0; q < 32; ++q) v[q] = 0.f;
            }
#pragma unroll
            for (int q = 0; q < 8; ++q)
                *reinterpret_cast<float4*>(smem + RED + red_off(row, half * 16 + c * 8 + q)) =
                    make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        float t = 0.f;
        for (int w = 0; w < kThreads / 32; ++w) t += wsum[w];
        wsum[10] = t / (float)T;
    }
    if (a.w_next && threadIdx.x == kLoadWarp * 32 && !*abort_word) {
        // the Delta products have completed: phi_q (for the next frame's W) into
        // the phi_v tile, as an MN-major A operand
        tma_prefetch_desc(&tm_phiq);
        mbar_expect_tx(&bars[B_WPHI], kTileBytes);
        tma_load_3d(sb + PHIV, &tm_phiq, &bars[B_WPHI], 0, 0, h);
        tma_load_3d(sb + PHIV + kHalf, &tm_phiq, &bars[B_WPHI], 64, 0, h);
        wphi_issued = true;
    }
    cluster_sync();  // every CTA of the cluster has parked Delta_c and staged S_{N-1}

    // ------------------------------------------------------------ reduce and apply this CTA's band
    // S_N[row] = alpha S_{N-1}[row] + sum_c Delta_c[row], ranks summed in order
    {
        const int band = (128 + C - 1) / C;
        const int r0 = min(128, split * band), r1 = min(128, r0 + band);
        const float alpha = wsum[10];
        const float* Sp = reinterpret_cast<const float*>(smem + SPREV);
        float* S = a.state + (size_t)bh * 128 * 128;
        const int items = (r1 - r0) * 32;
        bool bad = false;
        for (int it = threadIdx.x; it < items && park_ok; it += 2 * kThreads) {
            const int it2 = it + kThreads;
            const bool second = it2 < items;
            const int row0 = r0 + it / 32, q0 = it % 32;
            const int row1 = second ? r0 + it2 / 32 : row0, q1 = second ? it2 % 32 : q0;
            const uint32_t off0 = red_off(row0, q0), off1 = red_off(row1, q1);
            float4 v0[kMaxClusterRanks], v1[kMaxClusterRanks];
#pragma unroll
            for (int c = 0; c < kMaxClusterRanks; ++c)
                if (c < C) {
                    v0[c] = ld_cluster_f4(sb + RED + off0, (uint32_t)c);
                    v1[c] = ld_cluster_f4(sb + RED + off1, (uint32_t)c);
                }
            float4 s0 = *reinterpret_cast<const float4*>(Sp + row0 * 128 + q0 * 4);
            float4 s1 = *reinterpret_cast<const float4*>(Sp + row1 * 128 + q1 * 4);
            s0 = make_float4(alpha * s0.x, alpha * s0.y, alpha * s0.z, alpha * s0.w);
            s1 = make_float4(alpha * s1.x, alpha * s1.y, alpha * s1.z, alpha * s1.w);
#pragma unroll
            for (int c = 0; c < kMaxClusterRanks; ++c)
                if (c < C) {
                    s0.x += v0[c].x; s0.y += v0[c].y; s0.z += v0[c].z; s0.w += v0[c].w;
                    s1.x += v1[c].x; s1.y += v1[c].y; s1.z += v1[c].z; s1.w += v1[c].w;
                }
            *reinterpret_cast<float4*>(S + row0 * 128 + q0 * 4) = s0;
            bad |= !(isfinite(s0.x) && isfinite(s0.y) && isfinite(s0.z) && isfinite(s0.w));
            if (second) {
                *reinterpret_cast<float4*>(S + row1 * 128 + q1 * 4) = s1;
                bad |= !(isfinite(s1.x) && isfinite(s1.y) && isfinite(s1.z) && isfinite(s1.w));
            }
        }
        if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(a.flags, FLAG_NONFINITE);
    }
    cluster_sync();  // no CTA leaves while another still reads its shared memory
    tc_fence_after();
    if (a.w_next) {
        // W_{N+1} = phi_q^T S_N for the next frame of a multi-frame call, with the
        // prep kernel's operands and instruction sequence (so the same bits); every
        // CTA of the cluster computes all of W and writes the rows of its band.  The
        // cluster barrier above (release / acquire) makes every band of S_N visible.
        const int half = warp >> 2;
        const int row = (warp & 3) * 32 + lane;
        if (warp < 8) {
            const float4* Sg = reinterpret_cast<const float4*>(a.state + (size_t)bh * 128 * 128 + row * 128 + half * 64);
            float4 sv[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) sv[k] = __ldcg(Sg + k);
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const float4 v = sv[k];
                const __nv_bfloat162 h01 = __floats2bfloat162_rn(v.x, v.y);
                const __nv_bfloat162 h23 = __floats2bfloat162_rn(v.z, v.w);
                const uint2 hi = make_uint2(*reinterpret_cast<const uint32_t*>(&h01),
                                            *reinterpret_cast<const uint32_t*>(&h23));
                const uint2 lo = make_uint2(pack_bf16(v.x - __low2float(h01), v.y - __high2float(h01)),
                                            pack_bf16(v.z - __low2float(h23), v.w - __high2float(h23)));
                const uint32_t off = half * kHalf + sw128_offset(row, k >> 1) + (k & 1) * 8;
                *reinterpret_cast<uint2*>(smem + SH + off) = hi;
                *reinterpret_cast<uint2*>(smem + SL + off) = lo;
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (threadIdx.x == kMmaWarp * 32) {
            if (park_ok && mbar_wait(&bars[B_WPHI], 0, abort_word, a.flags)) {
                constexpr uint32_t ID_MNMN = idesc_bf16(128, 128, 1, 1);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16(tD, mnmajor_desc(sb + PHIV, kk), mnmajor_desc(sb + SH, kk), ID_MNMN, kk > 0);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16(tD, mnmajor_desc(sb + PHIV, kk), mnmajor_desc(sb + SL, kk), ID_MNMN, 1);
            }
            mma_commit(&bars[B_WMMA]);
        }
        if (warp < 8) {
            const bool w_ok =
                __all_sync(0xffffffffu, park_ok && mbar_wait(&bars[B_WMMA], 0, abort_word, a.flags));
            const int band = (128 + C - 1) / C;
            const int r0 = min(128, split * band), r1 = min(128, r0 + band);
            if (w_ok) {
                tc_fence_after();
                const uint32_t lrow = (uint32_t)((warp & 3) * 32) << 16;
                const size_t base = ((size_t)bh * 128 + row) * 128 + half * 64;
                __nv_bfloat16* wlo = a.w_next + (size_t)a.B * a.H * 128 * 128;
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    float x[32];
                    tmem_ld32(tD + lrow + half * 64 + c * 32, x);
                    tmem_ld_wait();
                    if (row >= r0 && row < r1) {
                        uint32_t hi[16], lo[16];
#pragma unroll
                        for (int q = 0; q < 16; ++q) {
                            const float w0 = x[2 * q] * 1.0f, w1 = x[2 * q + 1] * 1.0f;
                            const __nv_bfloat162 hv = __floats2bfloat162_rn(w0, w1);
                            hi[q] = *reinterpret_cast<const uint32_t*>(&hv);
                            lo[q] = pack_bf16(w0 - __low2float(hv), w1 - __high2float(hv));
                        }
                        uint4* dh = reinterpret_cast<uint4*>(a.w_next + base + c * 32);
                        uint4* dl = reinterpret_cast<uint4*>(wlo + base + c * 32);
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            dh[q] = make_uint4(hi[4 * q], hi[4 * q + 1], hi[4 * q + 2], hi[4 * q + 3]);
                            dl[q] = make_uint4(lo[4 * q], lo[4 * q + 1], lo[4 * q + 2], lo[4 * q + 3]);
                        }
                    }
                }
            }
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    // after a wait gave up, copies this CTA issued may still be landing
    if (park_issued) mbar_drain(&bars[B_PARK], 0, a.wait_ns);
    if (wphi_issued) mbar_drain(&bars[B_WPHI], 0, a.wait_ns);
    if (warp == kMmaWarp) {
        // every product this CTA issued completes before its TMEM is released
        // (after a wait gave up, some were issued without being waited for)
        if (lane == 0) {
            mma_commit(&bars[B_DRAIN]);
            mbar_drain(&bars[B_DRAIN], 0, a.wait_ns);
        }
        __syncwarp();
        tmem_dealloc(tmem, 512);
    }
    // when launched as a programmatic dependent of the attention kernel, complete
    // only after it: later work in the stream (the next prep, which rewrites the
    // W the attention kernel reads) stays ordered after both
    pdl_wait_primary();
    if (a.chain_flags) {
        // this CTA is done with the state (its band written, S_N read for W) and
        // the attention kernel before it has completed: release the next chained
        // update, which overwrites both the state and the W slot that kernel read
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0) st_release_gpu(a.chain_flags + (size_t)bh * kMaxClusterRanks + split, a.chain_set);
    }
}

// ============================================================== prep: W = phi_q^T S_{N-1}
// The inter-frame read O_inter = Q' S_{N-1} = (Q phi_q^T) S_{N-1} is regrouped as
// Q W with W = phi_q^T S_{N-1} (exact), so the attention kernel multiplies each
// query tile by one d x d matrix.  One CTA per (batch, head), 8 warps:
// phi_q arrives by TMA as an MN-major A operand (A[i][o] = phi_q[o][i]),
// S_{N-1} by one bulk copy; the warps split S into bf16 hi + lo MN-major B tiles,
// one thread issues W = phi_q^T S_hi + phi_q^T S_lo (16 MMAs, fp32 in TMEM), and
// the warps write W (times the inter-frame gain c of a weighted pass) back as
// the row-major bf16 hi + lo pair the attention kernel loads.
namespace prep {
constexpr uint32_t PHI = 0;
constexpr uint32_t SF = PHI + kTileBytes;          // S_{N-1} fp32 [128][128]
constexpr uint32_t SH = SF + 128 * 128 * 4;
constexpr uint32_t SL = SH + kTileBytes;
constexpr uint32_t BAR = SL + kTileBytes;          // 163,840
constexpr uint32_t SMEM = BAR + 64;
constexpr int kThreads = 256;
enum { B_PHI = 0, B_S, B_MMA, B_COUNT };
}  // namespace prep

__global__ void __launch_bounds__(prep::kThreads, 1)
    prep_tc_kernel(const __grid_constant__ LayerArgs a, const __grid_constant__ CUtensorMap tm_phiq) {
    using namespace prep;
    extern __shared__ __align__(1024) uint8_t smem[];
    if (smem_u32(smem) & 1023u) {
        if (threadIdx.x == 0) atomicOr(a.flags, FLAG_INTERNAL);
        return;
    }
    const uint32_t sb = smem_u32(smem);
    uint64_t* bars = (uint64_t*)(smem + BAR);
    uint32_t* tmem_slot = (uint32_t*)(bars + B_COUNT);
    volatile int* abort_word = (volatile int*)(tmem_slot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.y, b = blockIdx.z;
    const int bh = b * a.H + h;
    if (threadIdx.x == 0) {
        for (int i = 0; i < B_COUNT; ++i) mbar_init(&bars[i], 1);
        *abort_word = 0;
        fence_mbar_init();
        fence_async_smem();
        mbar_expect_tx(&bars[B_PHI], kTileBytes);
        tma_load_3d(sb + PHI, &tm_phiq, &bars[B_PHI], 0, 0, h);
        tma_load_3d(sb + PHI + kHalf, &tm_phiq, &bars[B_PHI], 64, 0, h);
    }
    if (warp == 0) tmem_alloc(tmem_slot, 128);
    // launched as a programmatic dependent: the previous kernel of the stream may
    // write the state, so wait for it before reading S_{N-1}
    pdl_wait_primary();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (threadIdx.x == 0) {
        mbar_expect_tx(&bars[B_S], 128 * 128 * 4);
        bulk_load(sb + SF, a.state + (size_t)bh * 128 * 128, 128 * 128 * 4, &bars[B_S]);
    }
    const bool s_ok = __all_sync(0xffffffffu, mbar_wait(&bars[B_S], 0, abort_word, a.flags, a.wait_ns));
    // S_{N-1} is in shared memory: only now may the attention kernel start, and
    // through it the delta update that overwrites the state in place (it is
    // launched once every attention CTA has started)
    __syncthreads();
    pdl_launch_dependents();
    const int half = warp >> 2;
    const int row = (warp & 3) * 32 + lane;
    if (s_ok) {
        // S row `row`, columns 64 half..+63: bf16 hi + lo into the MN-major B tiles
        const float4* Sp4 = reinterpret_cast<const float4*>(smem + SF) + row * 32 + half * 16;
#pragma unroll
        for (int k0 = 0; k0 < 16; ++k0) {
            const int k = (k0 + lane) & 15;
            const float4 v = Sp4[k];
            const __nv_bfloat162 h01 = __floats2bfloat162_rn(v.x, v.y);
            const __nv_bfloat162 h23 = __floats2bfloat162_rn(v.z, v.w);
            const uint2 hi = make_uint2(*reinterpret_cast<const uint32_t*>(&h01),
                                        *reinterpret_cast<const uint32_t*>(&h23));
            const uint2 lo = make_uint2(pack_bf16(v.x - __low2float(h01), v.y - __high2float(h01)),
                                        pack_bf16(v.z - __low2float(h23), v.w - __high2float(h23)));
            const uint32_t off = half * kHalf + sw128_offset(row, k >> 1) + (k & 1) * 8;
            *reinterpret_cast<uint2*>(smem + SH + off) = hi;
            *reinterpret_cast<uint2*>(smem + SL + off) = lo;
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (threadIdx.x == 0) {
        if (s_ok && mbar_wait(&bars[B_PHI], 0, abort_word, a.flags, a.wait_ns)) {
            constexpr uint32_t ID_MNMN = idesc_bf16(128, 128, 1, 1);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_bf16(tmem, mnmajor_desc(sb + PHI, kk), mnmajor_desc(sb + SH, kk), ID_MNMN, kk > 0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_bf16(tmem, mnmajor_desc(sb + PHI, kk), mnmajor_desc(sb + SL, kk), ID_MNMN, 1);
        }
        mma_commit(&bars[B_MMA]);  // also when nothing was issued: the waiters below return
    }
    bool m_ok = __all_sync(0xffffffffu, s_ok && mbar_wait(&bars[B_MMA], 0, abort_word, a.flags, a.wait_ns));
    __syncthreads();
    m_ok = m_ok && *abort_word == 0;  // thread 0's wait for phi_q may have failed
    if (m_ok) {
        tc_fence_after();
        // W row `row` (TMEM lane), columns 64 half..+63 -> bf16 hi + lo, row-major
        const uint32_t lrow = (uint32_t)((warp & 3) * 32) << 16;
        const float cg = a.mix ? a.mix[bh * 2 + 1] : 1.0f;
        const size_t base = ((size_t)bh * 128 + row) * 128 + half * 64;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            float x[32];
            tmem_ld32(tmem + lrow + half * 64 + c * 32, x);
            tmem_ld_wait();
            uint32_t hi[16], lo[16];
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                const float w0 = x[2 * q] * cg, w1 = x[2 * q + 1] * cg;
                const __nv_bfloat162 hv = __floats2bfloat162_rn(w0, w1);
                hi[q] = *reinterpret_cast<const uint32_t*>(&hv);
                lo[q] = pack_bf16(w0 - __low2float(hv), w1 - __high2float(hv));
            }
            uint4* dh = reinterpret_cast<uint4*>(a.WT_hi + base + c * 32);
            uint4* dl = reinterpret_cast<uint4*>(a.WT_lo + base + c * 32);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                dh[q] = make_uint4(hi[4 * q], hi[4 * q + 1], hi[4 * q + 2], hi[4 * q + 3]);
                dl[q] = make_uint4(lo[4 * q], lo[4 * q + 1], lo[4 * q + 2], lo[4 * q + 3]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 128);
}

}  // namespace tc
}  // namespace hyb
