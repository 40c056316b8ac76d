// hyb_attn.cu -- C ABI of the ARL2 hybrid attention layer: argument checks,
// workspace plan and the launch sequence of one pass.
//
// Source: "Technical summary: Attend Locally, Remember Linearly (ARL2)",
// gist.science/ar/paper/2605.16579, §2.1 and §2.2; the interface contract is
// documented in include/hyb_attn.h.
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <new>

#include "hyb_attn.h"
#include "common.cuh"
#include "simt_layer.cuh"
#include "tc_kernels.cuh"
#include "tc_attention.cuh"
#include "token_level.cuh"
#include "tra.cuh"

namespace {

using namespace hyb;

constexpr int kMaxDevices = 64;

struct Plan {
    int D;
    bool bf16;
    int nsplit;
    int split_tokens;
    size_t off_W, off_Sprev, off_part, off_chain, total;
};

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Token splits of the state update: about `want` splits of whole 128-token
// tiles (at most one cluster's worth on the tensor path).
void update_split(int T, int want, bool bf16, int* nsplit, int* split_tokens) {
    const int ntiles = (T + kUpdateTile - 1) / kUpdateTile;
    if (bf16 && want > tc::kMaxClusterRanks) want = tc::kMaxClusterRanks;
    if (want > ntiles) want = ntiles;
    if (want < 1) want = 1;
    const int tiles_per_split = (ntiles + want - 1) / want;
    *split_tokens = tiles_per_split * kUpdateTile;
    *nsplit = (ntiles + tiles_per_split - 1) / tiles_per_split;
}

hyb_status make_plan(const hyb_attn_desc* d, Plan* p) {
    if (!d) return HYB_ERR_INVALID;
    if (d->B <= 0 || d->H <= 0 || d->T <= 0 || d->d_k <= 0 || d->d_v <= 0) return HYB_ERR_INVALID;
    if (d->dtype != HYB_BF16 && d->dtype != HYB_FP32) return HYB_ERR_INVALID;
    if (!(d->l2_eps >= 0.f) || !isfinite(d->l2_eps) || !isfinite(d->sm_scale)) return HYB_ERR_INVALID;
    if (d->d_k != d->d_v) return HYB_ERR_UNSUPPORTED;
    const int D = d->d_k;
    const bool bf16 = d->dtype == HYB_BF16;
    if (!((bf16 && D == 128) || (!bf16 && D == 32))) return HYB_ERR_UNSUPPORTED;
    if (d->H > 65535 || d->B > 65535) return HYB_ERR_UNSUPPORTED;
    const double elems = (double)d->B * d->T * d->H * D;
    if (elems >= 2147483647.0) return HYB_ERR_UNSUPPORTED;
    p->D = D;
    p->bf16 = bf16;
    // token splits of the state update, each a whole number of 128-token tiles.
    // Tensor path: one cluster of at most 8 CTAs per (b, h), splits reduced in
    // distributed shared memory (no partials in the workspace).  The update runs
    // beside attention kernels (the second wave of its own frame's, or the next
    // frame's), so its splits take about a quarter of the SMs in all and at least
    // 3 per head: fewer CTAs per head cost less SM time for the same work, more
    // shorten the chain from one frame's state to the next (which consecutive
    // updates of a frames call overlap).  fp32 path: enough (b, h, split) blocks
    // to cover the SMs, partials in the workspace.
    const int BH = d->B * d->H;
    const int quarter = kNumSMs / (4 * BH) > 3 ? kNumSMs / (4 * BH) : 3;
    update_split(d->T, bf16 ? quarter : (kNumSMs + BH - 1) / BH, bf16, &p->nsplit, &p->split_tokens);
    const size_t hh = (size_t)BH * D * D;
    p->off_W = kStatusBytes;
    // fp32 W, or the two bf16 halves of W; then the fp32 path's copy of S_{N-1},
    // which on the tensor path is the second W slot of chained passes
    p->off_Sprev = align_up(p->off_W + hh * sizeof(float), 256);
    p->off_part = align_up(p->off_Sprev + hh * sizeof(float), 256);
    // fp32 path: split partials (the tensor path reduces its splits on chip)
    const size_t part_bytes = bf16 ? 0 : hh * 2 * p->nsplit * sizeof(float);
    // chained passes: one flag word per update CTA (a cluster of at most 8 per head)
    p->off_chain = align_up(p->off_part + part_bytes, 256);
    p->total = align_up(p->off_chain + (size_t)BH * tc::kMaxClusterRanks * sizeof(unsigned), 256);
    return HYB_OK;
}

// ---- optional kernel timing -------------------------------------------------
enum { K_PREP = 0, K_ATTN = 1, K_UPDATE = 2, K_APPLY = 3, K_TOK_PREP = 4, K_TOK_CHAIN = 5, K_TOK_READS = 6 };

struct Timing {
    bool on = false;
    int cap = 0, used = 0, dropped = 0;
    cudaEvent_t* ev = nullptr;   // 2 * cap events: start, stop per launch
    int* kind = nullptr;
} g_timing;

// Launch through `fn`, bracketed by timing events when timing is on.
template <typename F>
cudaError_t timed(int kind, cudaStream_t st, F fn) {
    if (!g_timing.on) {
        fn();
        return cudaSuccess;
    }
    if (g_timing.used >= g_timing.cap) {
        ++g_timing.dropped;
        fn();
        return cudaSuccess;
    }
    const int i = g_timing.used++;
    g_timing.kind[i] = kind;
    cudaError_t e = cudaEventRecord(g_timing.ev[2 * i], st);
    fn();
    if (e == cudaSuccess) e = cudaEventRecord(g_timing.ev[2 * i + 1], st);
    return e;
}

bool aligned16(const void* ptr) { return ((uintptr_t)ptr & 15u) == 0; }

// Fault test (off by default): see hyb_attn_set_fault_test in the header.
struct FaultTest {
    int skip_v = 0;
    unsigned long long wait_ns = 2000000000ull;
} g_fault;

// Opt each kernel into its dynamic shared memory once per device.
template <typename K>
cudaError_t opt_in_smem(K kernel, size_t bytes, unsigned char* done) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    if (done[dev]) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    // every kernel of a pass asks for the same (largest) shared-memory carveout, so
    // an SM freed by one kernel takes the next one's CTAs without reconfiguring
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 (int)cudaSharedmemCarveoutMaxShared);
    if (e == cudaSuccess) done[dev] = 1;
    return e;
}

// CTAs of the attention kernel along the query axis: one per 128-query tile.
unsigned attn_tiles(int T) { return (unsigned)((T + tc::kTile - 1) / tc::kTile); }

// Query tiles per attention CTA for a chained pass: two when one tile per CTA
// would take more than one wave of the SMs but at most two (the second nearly
// empty for a 480p frame), so the grid fits one wave and leaves SMs to the delta
// update that runs beside it; one otherwise, and for block-sparse and entropy
// passes (whose CTAs take one listed tile each).  (A CTA runs its tiles one
// after another, so an attention kernel alone gains nothing from this, and a
// frames call, which packs consecutive frames' kernels, runs one tile per CTA.)
int attn_q_per_cta(const LayerArgs& a) {
    const long long tiles = (long long)attn_tiles(a.T) * a.H * a.B;
    const int key_tiles = (a.T_kv + tc::kTile - 1) / tc::kTile;
    if (a.kv_list || a.kv_order || a.ent_out || !a.inter || key_tiles < 3) return 1;
    return tiles > kNumSMs && tiles <= 2 * kNumSMs ? 2 : 1;
}

template <int D, typename TIO>
cudaError_t launch_simt(const LayerArgs& a, int clean, cudaStream_t st) {
    static unsigned char done_prep[kMaxDevices], done_attn[kMaxDevices], done_part[kMaxDevices],
        done_apply[kMaxDevices];
    cudaError_t e;
    const dim3 rows(D / simt::prep_rows<false>(), a.H, a.B);
    const size_t prep_smem = simt::PrepSmem<D, simt::prep_rows<false>()>::bytes;
    const size_t attn_smem = simt::AttnSmem<D>::bytes;
    const size_t ps = simt::PartialsSmem<D>::bytes;
    const size_t as = simt::ApplySmem<D, TIO>::bytes;
    if ((e = opt_in_smem(simt::prep_kernel<D, TIO, false>, prep_smem, done_prep)) != cudaSuccess) return e;
    if ((e = opt_in_smem(simt::attn_kernel<D, TIO>, attn_smem, done_attn)) != cudaSuccess) return e;
    if ((e = opt_in_smem(simt::partials_kernel<D, TIO>, ps, done_part)) != cudaSuccess) return e;
    if ((e = opt_in_smem(simt::apply_kernel<D, TIO>, as, done_apply)) != cudaSuccess) return e;
    e = timed(K_PREP, st, [&] {
        simt::prep_kernel<D, TIO, false><<<rows, simt::kThreads, prep_smem, st>>>(a, clean);
    });
    if (e != cudaSuccess) return e;
    const dim3 agrid((a.T + simt::AttnSmem<D>::BQ - 1) / simt::AttnSmem<D>::BQ, a.H, a.B);
    e = timed(K_ATTN, st, [&] { simt::attn_kernel<D, TIO><<<agrid, simt::kThreads, attn_smem, st>>>(a); });
    if (e != cudaSuccess) return e;
    if (clean) {
        e = timed(K_UPDATE, st, [&] {
            simt::partials_kernel<D, TIO><<<dim3(a.nsplit, a.H, a.B), simt::kThreads, ps, st>>>(a);
        });
        if (e != cudaSuccess) return e;
        e = timed(K_APPLY, st, [&] { simt::apply_kernel<D, TIO><<<rows, simt::kThreads, as, st>>>(a); });
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

// ---- tensor-core path (bf16, d = 128) ----------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (EncodeTiledFn)p;
    }
    return fn;
}

// Encoded tensor maps of recent calls, per host thread: a frame loop passes
// the same buffers again and again, so most calls find every map here and
// skip the driver's encoder.  The key is everything the encoding depends on.
struct MapKey {
    const void* base;
    uint64_t d0, d1, d2, s1, s2;
    bool operator==(const MapKey& o) const {
        return base == o.base && d0 == o.d0 && d1 == o.d1 && d2 == o.d2 && s1 == o.s1 && s2 == o.s2;
    }
};
struct MapCache {
    static constexpr int kEntries = 128;
    MapKey key[kEntries];
    CUtensorMap map[kEntries];
    int used = 0, next = 0;
};
thread_local MapCache t_maps;

// 3-D bf16 tensor map with 64 x 128 x 1 boxes and 128-byte swizzle:
// dims {d0 (contiguous), d1, d2}, byte strides s1, s2 of dims 1 and 2.
bool map3d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1,
           uint64_t s2) {
    const MapKey k = {base, d0, d1, d2, s1, s2};
    MapCache& c = t_maps;
    for (int i = 0; i < c.used; ++i)
        if (c.key[i] == k) {
            *m = c.map[i];
            return true;
        }
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {s1, s2};
    cuuint32_t box[3] = {64, 128, 1};
    cuuint32_t es[3] = {1, 1, 1};
    if (fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    const int slot = c.used < MapCache::kEntries ? c.used++ : c.next++ % MapCache::kEntries;
    c.key[slot] = k;
    c.map[slot] = *m;
    return true;
}

// The three kernels of one bf16 pass: tensor maps encoded once, each kernel
// launchable on a given stream, as a programmatic dependent of the previous
// kernel of that stream or not.
struct TcPass {
    LayerArgs a;
    CUtensorMap tq, tk, tv, tw, tphik, tphiq, tout;

    cudaError_t init(const LayerArgs& args) {
        static unsigned char done_prep[kMaxDevices], done_attn[kMaxDevices], done_upd[kMaxDevices];
        constexpr int D = 128;
        a = args;
        a.q_per_cta = 1;
        cudaError_t e;
        if ((e = opt_in_smem(tc::prep_tc_kernel, tc::prep::SMEM, done_prep)) != cudaSuccess) return e;
        static unsigned char done_attn_ent[kMaxDevices], done_attn_multi[kMaxDevices];
        if ((e = opt_in_smem(tc::attention_kernel<false>, tc::attn::SMEM, done_attn)) != cudaSuccess) return e;
        if ((e = opt_in_smem(tc::attention_kernel<true>, tc::attn::SMEM, done_attn_ent)) != cudaSuccess) return e;
        if ((e = opt_in_smem(tc::attention_kernel<false, true>, tc::attn::SMEM, done_attn_multi)) != cudaSuccess)
            return e;
        if ((e = opt_in_smem(tc::update_kernel, tc::upd::SMEM, done_upd)) != cudaSuccess) return e;
        const uint64_t row_bytes = (uint64_t)a.H * D * 2;
        const uint64_t bh = (uint64_t)a.B * a.H;
        if (!map3d(&tq, a.q, (uint64_t)a.H * D, a.T, a.B, row_bytes, row_bytes * a.T) ||
            (a.out && !map3d(&tout, a.out, (uint64_t)a.H * D, a.T, a.B, row_bytes, row_bytes * a.T)) ||
            !map3d(&tk, a.k, (uint64_t)a.H * D, a.T, a.B, row_bytes, row_bytes * a.T) ||
            !map3d(&tv, a.v, (uint64_t)a.H * D, a.T, a.B, row_bytes, row_bytes * a.T) ||
            !map3d(&tw, a.WT_hi, D, D, 2 * bh, D * 2, D * D * 2) ||
            !map3d(&tphik, a.phi_k, D, D, a.H, D * 2, D * D * 2) ||
            !map3d(&tphiq, a.phi_q, D, D, a.H, D * 2, D * D * 2))
            return cudaErrorInvalidValue;
        if (!a.out) tout = tq;  // not read: the attention kernel stores no bf16 output
        return cudaSuccess;
    }

    static void pdl_attr(cudaLaunchAttribute* at) {
        at->id = cudaLaunchAttributeProgrammaticStreamSerialization;
        at->val.programmaticStreamSerializationAllowed = 1;
    }

    cudaError_t prep(cudaStream_t st, bool pdl) {
        cudaLaunchAttribute at[1];
        pdl_attr(&at[0]);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(1, a.H, a.B);
        cfg.blockDim = dim3(tc::prep::kThreads, 1, 1);
        cfg.dynamicSmemBytes = tc::prep::SMEM;
        cfg.stream = st;
        cfg.attrs = at;
        cfg.numAttrs = pdl ? 1 : 0;
        cudaError_t le = cudaSuccess;
        cudaError_t e = timed(K_PREP, st, [&] { le = cudaLaunchKernelEx(&cfg, tc::prep_tc_kernel, a, tphiq); });
        return e != cudaSuccess ? e : le;
    }

    cudaError_t attn(cudaStream_t st, bool pdl) {
        cudaLaunchAttribute at[1];
        pdl_attr(&at[0]);
        cudaLaunchConfig_t cfg = {};
        const unsigned qpc = a.q_per_cta > 1 ? (unsigned)a.q_per_cta : 1u;
        cfg.gridDim = dim3((attn_tiles(a.T) + qpc - 1) / qpc, a.H, a.B);
        cfg.blockDim = dim3(tc::attn::kThreads, 1, 1);
        cfg.dynamicSmemBytes = tc::attn::SMEM;
        cfg.stream = st;
        cfg.attrs = at;
        cfg.numAttrs = pdl ? 1 : 0;
        cudaError_t le = cudaSuccess;
        // the entropy-writing variant for the warm-up pass of Token Radius Attention
        cudaError_t e = timed(K_ATTN, st, [&] {
            le = a.ent_out       ? cudaLaunchKernelEx(&cfg, tc::attention_kernel<true>, a, tq, tk, tv, tw, tout)
                 : qpc > 1       ? cudaLaunchKernelEx(&cfg, tc::attention_kernel<false, true>, a, tq, tk, tv, tw, tout)
                                 : cudaLaunchKernelEx(&cfg, tc::attention_kernel<false>, a, tq, tk, tv, tw, tout);
        });
        return e != cudaSuccess ? e : le;
    }

    cudaError_t update(cudaStream_t st, bool pdl) {
        // one cluster of nsplit CTAs per (b, h)
        cudaLaunchAttribute at[2];
        at[0].id = cudaLaunchAttributeClusterDimension;
        at[0].val.clusterDim.x = a.nsplit;
        at[0].val.clusterDim.y = 1;
        at[0].val.clusterDim.z = 1;
        pdl_attr(&at[1]);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(a.nsplit, a.H, a.B);
        cfg.blockDim = dim3(tc::upd::kThreads, 1, 1);
        cfg.dynamicSmemBytes = tc::upd::SMEM;
        cfg.stream = st;
        cfg.attrs = at;
        cfg.numAttrs = pdl ? 2 : 1;
        cudaError_t le = cudaSuccess;
        cudaError_t e = timed(K_UPDATE, st, [&] {
            le = cudaLaunchKernelEx(&cfg, tc::update_kernel, a, tk, tv, tphik, tphiq);
        });
        return e != cudaSuccess ? e : le;
    }
};

cudaError_t launch_tc(const LayerArgs& a, int clean, cudaStream_t st) {
    TcPass tp;
    cudaError_t e = tp.init(a);
    if (e != cudaSuccess) return e;
    // Kernels of a pass are chained by programmatic dependent launch: prep waits
    // for the previous kernel of the stream and stages the state, then lets the
    // attention kernel start (which reads prep's W only at its end, after waiting
    // for prep); the delta update starts once every attention CTA has started (on
    // the SMs the last wave leaves idle), so after prep has read the state it
    // overwrites, and completes only after the attention grid.
    if ((e = tp.prep(st, true)) != cudaSuccess) return e;
    if ((e = tp.attn(st, true)) != cudaSuccess) return e;
    if (clean && (e = tp.update(st, true)) != cudaSuccess) return e;
    return cudaGetLastError();
}

// ---- chained passes -----------------------------------------------------------
// What hyb_attn_forward_next knows about a workspace after its last pass there:
// the pass's buffers and stream, the W slot that holds phi_q^T of the present
// state, and the flag value the last chained delta update on this state sets
// (0: none since the chain's prep).  Any other pass on the workspace or the
// state drops the record, so the next chained call starts over with prep.
struct ChainRec {
    const void* ws = nullptr;  // null: free entry
    const float* state;
    const void* phi_q;
    cudaStream_t stream;
    int B, H, T, dtype, d;
    float sm_scale, l2_eps;
    int cur;
    unsigned epoch;
};
constexpr int kChainRecs = 16;
ChainRec g_chain[kChainRecs];
unsigned g_chain_epoch = 0;
int g_chain_victim = 0;

void chain_forget(const void* ws, const float* state) {
    for (ChainRec& r : g_chain)
        if (r.ws && (r.ws == ws || (state && r.state == state))) r.ws = nullptr;
}

bool chain_find(const void* ws, ChainRec* out) {
    for (const ChainRec& r : g_chain)
        if (r.ws && r.ws == ws) {
            *out = r;
            return true;
        }
    return false;
}

void chain_store(const ChainRec& rec) {
    for (ChainRec& r : g_chain)
        if (!r.ws) {
            r = rec;
            return;
        }
    g_chain[g_chain_victim] = rec;
    g_chain_victim = (g_chain_victim + 1) % kChainRecs;
}

unsigned chain_next_epoch() {
    if (++g_chain_epoch == 0) ++g_chain_epoch;
    return g_chain_epoch;
}

// Checks every argument of a pass and fills the kernels' argument block;
// enqueues nothing, so an error here leaves the stream untouched.  A pass on a
// workspace or a state ends any chain of passes that used them.
hyb_status pass_args(const hyb_attn_desc* desc, const void* q, const void* k, const void* v,
                     const void* phi_q, const void* phi_k, const void* phi_v, const float* gate_logits,
                     const float* beta_logits, float* state, int clean_pass, void* out, float* out_intra,
                     float* out_inter, void* workspace, size_t workspace_bytes, const float* mix,
                     LayerArgs* args, Plan* plan) {
    Plan p;
    hyb_status s = make_plan(desc, &p);
    if (s != HYB_OK) return s;
    if (clean_pass != 0 && clean_pass != 1) return HYB_ERR_INVALID;
    if (!q || !k || !v || !phi_q || !phi_k || !phi_v || !state) return HYB_ERR_INVALID;
    if (!out && !(out_intra && out_inter)) return HYB_ERR_INVALID;
    if ((out_intra == nullptr) != (out_inter == nullptr)) return HYB_ERR_INVALID;
    if (clean_pass && (!gate_logits || !beta_logits)) return HYB_ERR_INVALID;
    const void* ptrs[] = {q, k, v, phi_q, phi_k, phi_v, state, out, out_intra, out_inter,
                          gate_logits, beta_logits, workspace, mix};
    for (const void* ptr : ptrs)
        if (ptr && !aligned16(ptr)) return HYB_ERR_ALIGN;
    if (!workspace || workspace_bytes < p.total) return HYB_ERR_WORKSPACE;
    chain_forget(workspace, state);

    LayerArgs a;
    memset(&a, 0, sizeof(a));
    a.B = desc->B;
    a.H = desc->H;
    a.T = desc->T;
    a.T_kv = desc->T;
    a.inter = 1;
    a.mix = mix;
    a.D = p.D;
    const float scale = desc->sm_scale > 0.f ? desc->sm_scale : 1.0f / sqrtf((float)desc->d_k);
    a.sm_scale_log2 = scale * 1.4426950408889634f;
    a.l2_eps = desc->l2_eps;
    a.q = q;
    a.k = k;
    a.v = v;
    a.phi_q = phi_q;
    a.phi_k = phi_k;
    a.phi_v = phi_v;
    a.gate_logits = gate_logits;
    a.beta_logits = beta_logits;
    a.state = state;
    a.out = out;
    a.out_intra = out_intra;
    a.out_inter = out_inter;
    char* ws = (char*)workspace;
    a.flags = (unsigned*)ws;
    a.W = (float*)(ws + p.off_W);
    a.WT_hi = (__nv_bfloat16*)(ws + p.off_W);
    a.WT_lo = a.WT_hi + (size_t)a.B * a.H * p.D * p.D;
    a.S_prev = (float*)(ws + p.off_Sprev);
    a.partials = (float*)(ws + p.off_part);
    a.nsplit = p.nsplit;
    a.split_tokens = p.split_tokens;
    a.wait_ns = g_fault.wait_ns;
    a.dbg_skip_v = g_fault.skip_v;
    *args = a;
    *plan = p;
    return HYB_OK;
}

// ---- token-level access (clean passes) -------------------------------------------
struct TokPlan {
    size_t off_rec, off_out, total;
    int nch;
};

TokPlan tok_plan(const hyb_attn_desc* d, const Plan& p) {
    TokPlan t;
    t.nch = (d->T + tok::kChunk - 1) / tok::kChunk;
    const size_t rec_floats = p.D == 128 ? tok::Rec<128>::floats : tok::Rec<32>::floats;
    const size_t recs = (size_t)d->B * d->H * t.nch * rec_floats * sizeof(float);
    t.off_rec = align_up(p.total, 256);
    t.off_out = align_up(t.off_rec + recs, 256);
    t.total = align_up(t.off_out + (size_t)d->B * d->T * d->H * p.D * sizeof(float), 256);
    return t;
}

template <int D, typename TIO>
cudaError_t launch_token_level(LayerArgs a, const TokPlan& tp, char* ws, cudaStream_t st) {
    static unsigned char done_prep[kMaxDevices], done_chain[kMaxDevices], done_reads[kMaxDevices];
    cudaError_t e;
    if ((e = opt_in_smem(tok::chunk_prep_kernel<D, TIO>, tok::PrepSmem<D>::bytes, done_prep)) != cudaSuccess) return e;
    if ((e = opt_in_smem(tok::chunk_chain_kernel<D>, tok::ChainSmem<D>::bytes, done_chain)) != cudaSuccess) return e;
    if ((e = opt_in_smem(tok::chunk_reads_kernel<D>, tok::ReadsSmem<D>::bytes, done_reads)) != cudaSuccess) return e;
    float* rec = (float*)(ws + tp.off_rec);
    float* oi = (float*)(ws + tp.off_out);
    const dim3 cg(tp.nch, a.H, a.B);
    e = timed(K_TOK_PREP, st, [&] {
        tok::chunk_prep_kernel<D, TIO><<<cg, tok::kThreads, tok::PrepSmem<D>::bytes, st>>>(a, rec);
    });
    if (e != cudaSuccess) return e;
    e = timed(K_TOK_CHAIN, st, [&] {
        tok::chunk_chain_kernel<D><<<dim3(D / tok::kBand, a.H, a.B), D, tok::ChainSmem<D>::bytes, st>>>(a, rec);
    });
    if (e != cudaSuccess) return e;
    e = timed(K_TOK_READS, st, [&] {
        tok::chunk_reads_kernel<D><<<cg, tok::kThreads, tok::ReadsSmem<D>::bytes, st>>>(a, rec, oi);
    });
    if (e != cudaSuccess) return e;
    // the attention kernel adds the token-level read instead of Q W
    a.inter = 0;
    a.oi_ext = oi;
    if constexpr (D == 128) {
        static unsigned char done_attn[kMaxDevices];
        if ((e = opt_in_smem(tc::attention_kernel<false>, tc::attn::SMEM, done_attn)) != cudaSuccess) return e;
        const uint64_t row_bytes = (uint64_t)a.H * D * 2;
        CUtensorMap tq, tk, tv, tout;
        if (!map3d(&tq, a.q, (uint64_t)a.H * D, a.T, a.B, row_bytes, row_bytes * a.T) ||
            !map3d(&tk, a.k, (uint64_t)a.H * D, a.T, a.B, row_bytes, row_bytes * a.T) ||
            !map3d(&tv, a.v, (uint64_t)a.H * D, a.T, a.B, row_bytes, row_bytes * a.T) ||
            (a.out && !map3d(&tout, a.out, (uint64_t)a.H * D, a.T, a.B, row_bytes, row_bytes * a.T)))
            return cudaErrorInvalidValue;
        if (!a.out) tout = tq;
        cudaLaunchConfig_t acfg = {};
        acfg.gridDim = dim3(attn_tiles(a.T), a.H, a.B);
        acfg.blockDim = dim3(tc::attn::kThreads, 1, 1);
        acfg.dynamicSmemBytes = tc::attn::SMEM;
        acfg.stream = st;
        cudaError_t le = cudaSuccess;
        // tq stands in for the unused W map
        e = timed(K_ATTN, st,
                  [&] { le = cudaLaunchKernelEx(&acfg, tc::attention_kernel<false>, a, tq, tk, tv, tq, tout); });
        if (e != cudaSuccess) return e;
        if (le != cudaSuccess) return le;
    } else {
        static unsigned char done_attn[kMaxDevices];
        const size_t attn_smem = simt::AttnSmem<D>::bytes;
        if ((e = opt_in_smem(simt::attn_kernel<D, TIO>, attn_smem, done_attn)) != cudaSuccess) return e;
        const dim3 agrid((a.T + simt::AttnSmem<D>::BQ - 1) / simt::AttnSmem<D>::BQ, a.H, a.B);
        e = timed(K_ATTN, st, [&] { simt::attn_kernel<D, TIO><<<agrid, simt::kThreads, attn_smem, st>>>(a); });
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

hyb_status launch_pass(const LayerArgs& a, const Plan& p, int clean_pass, void* stream) {
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e;
    if (p.bf16)
        e = launch_tc(a, clean_pass, st);
    else
        e = launch_simt<32, float>(a, clean_pass, st);
    return e == cudaSuccess ? HYB_OK : HYB_ERR_CUDA;
}

// ---- several frames in one call ---------------------------------------------------
// Per device: a high-priority stream for the state chain (prep, update of each
// frame), a stream for the attention kernels, and events; created on the first
// call on the device and kept.  The calls are not thread-safe.
constexpr int kAttStreams = 2;  // attention kernels of consecutive frames alternate between them
struct FrameRes {
    bool ready = false;
    cudaStream_t chain = nullptr, att[kAttStreams] = {};
    cudaEvent_t fork = nullptr, join_chain = nullptr, join_att[kAttStreams] = {};
    cudaEvent_t* w = nullptr;
    int nw = 0;
};
FrameRes g_frames[kMaxDevices];
constexpr int kMaxFrames = 4096;

cudaError_t frame_resources(int n, FrameRes** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    FrameRes& r = g_frames[dev];
    if (!r.ready) {
        int least = 0, greatest = 0;
        if ((e = cudaDeviceGetStreamPriorityRange(&least, &greatest)) != cudaSuccess) return e;
        if ((e = cudaStreamCreateWithPriority(&r.chain, cudaStreamNonBlocking, greatest)) != cudaSuccess) return e;
        for (int i = 0; i < kAttStreams; ++i) {
            if ((e = cudaStreamCreateWithPriority(&r.att[i], cudaStreamNonBlocking, least)) != cudaSuccess) return e;
            if ((e = cudaEventCreateWithFlags(&r.join_att[i], cudaEventDisableTiming)) != cudaSuccess) return e;
        }
        if ((e = cudaEventCreateWithFlags(&r.fork, cudaEventDisableTiming)) != cudaSuccess) return e;
        if ((e = cudaEventCreateWithFlags(&r.join_chain, cudaEventDisableTiming)) != cudaSuccess) return e;
        r.ready = true;
    }
    if (r.nw < n) {
        cudaEvent_t* w = new (std::nothrow) cudaEvent_t[n];
        if (!w) return cudaErrorMemoryAllocation;
        int made = 0;
        for (; made < n; ++made)
            if ((e = cudaEventCreateWithFlags(&w[made], cudaEventDisableTiming)) != cudaSuccess) break;
        if (made < n) {
            for (int i = 0; i < made; ++i) cudaEventDestroy(w[i]);
            delete[] w;
            return e;
        }
        // events of earlier calls: the waits on them were enqueued by those calls
        for (int i = 0; i < r.nw; ++i) cudaEventDestroy(r.w[i]);
        delete[] r.w;
        r.w = w;
        r.nw = n;
    }
    *out = &r;
    return cudaSuccess;
}

size_t frames_w_bytes(const hyb_attn_desc* d, const Plan& p) {
    return (size_t)d->B * d->H * p.D * p.D * 2 * sizeof(__nv_bfloat16);
}

size_t frames_total(const hyb_attn_desc* d, const Plan& p, int n) {
    return align_up(p.total, 256) + (p.bf16 ? (size_t)n * align_up(frames_w_bytes(d, p), 256) : 0);
}

hyb_status forward_impl(const hyb_attn_desc* desc, const void* q, const void* k, const void* v,
                        const void* phi_q, const void* phi_k, const void* phi_v,
                        const float* gate_logits, const float* beta_logits, float* state,
                        int clean_pass, void* out, float* out_intra, float* out_inter,
                        void* workspace, size_t workspace_bytes, void* stream, const float* mix = nullptr) {
    LayerArgs a;
    Plan p;
    hyb_status s = pass_args(desc, q, k, v, phi_q, phi_k, phi_v, gate_logits, beta_logits, state, clean_pass,
                             out, out_intra, out_inter, workspace, workspace_bytes, mix, &a, &p);
    if (s != HYB_OK) return s;
    return launch_pass(a, p, clean_pass, stream);
}

// Softmax attention of one frame's queries over a KV cache (the baseline the
// hybrid layer replaces): append the frame's k, v at row `cached` of each
// batch's cache, then run the attention kernel over cached + T keys with no
// inter-frame read.
hyb_status kvcache_impl(const hyb_attn_desc* desc, const void* q, const void* k, const void* v, void* k_cache,
                        void* v_cache, int cache_tokens, int cached_tokens, void* out, void* workspace,
                        size_t workspace_bytes, void* stream) {
    if (!desc) return HYB_ERR_INVALID;
    if (desc->B <= 0 || desc->H <= 0 || desc->T <= 0 || desc->d_k <= 0 || desc->d_v <= 0) return HYB_ERR_INVALID;
    if (desc->dtype != HYB_BF16 && desc->dtype != HYB_FP32) return HYB_ERR_INVALID;
    if (!isfinite(desc->sm_scale)) return HYB_ERR_INVALID;
    if (desc->dtype != HYB_BF16 || desc->d_k != 128 || desc->d_v != 128) return HYB_ERR_UNSUPPORTED;
    if (desc->H > 65535 || desc->B > 65535) return HYB_ERR_UNSUPPORTED;
    if (cached_tokens < 0 || cache_tokens <= 0 || (long long)cached_tokens + desc->T > cache_tokens)
        return HYB_ERR_INVALID;
    if ((double)desc->B * cache_tokens * desc->H * 128 >= 2147483647.0) return HYB_ERR_UNSUPPORTED;
    if (!q || !k || !v || !k_cache || !v_cache || !out) return HYB_ERR_INVALID;
    const void* ptrs[] = {q, k, v, k_cache, v_cache, out, workspace};
    for (const void* ptr : ptrs)
        if (ptr && !aligned16(ptr)) return HYB_ERR_ALIGN;
    if (!workspace || workspace_bytes < kStatusBytes) return HYB_ERR_WORKSPACE;
    chain_forget(workspace, nullptr);

    constexpr int D = 128;
    const int B = desc->B, H = desc->H, T = desc->T;
    cudaStream_t st = (cudaStream_t)stream;
    const size_t row = (size_t)H * D;  // elements per token row
    for (int b = 0; b < B; ++b) {
        const size_t dst = ((size_t)b * cache_tokens + cached_tokens) * row * 2;
        const size_t src = (size_t)b * T * row * 2;
        if (cudaMemcpyAsync((char*)k_cache + dst, (const char*)k + src, (size_t)T * row * 2,
                            cudaMemcpyDeviceToDevice, st) != cudaSuccess ||
            cudaMemcpyAsync((char*)v_cache + dst, (const char*)v + src, (size_t)T * row * 2,
                            cudaMemcpyDeviceToDevice, st) != cudaSuccess)
            return HYB_ERR_CUDA;
    }
    LayerArgs a;
    memset(&a, 0, sizeof(a));
    a.B = B;
    a.H = H;
    a.T = T;
    a.T_kv = cached_tokens + T;
    a.inter = 0;
    a.D = D;
    const float scale = desc->sm_scale > 0.f ? desc->sm_scale : 1.0f / sqrtf((float)desc->d_k);
    a.sm_scale_log2 = scale * 1.4426950408889634f;
    a.q = q;
    a.k = k_cache;
    a.v = v_cache;
    a.out = out;
    a.flags = (unsigned*)workspace;
    a.wait_ns = g_fault.wait_ns;
    a.dbg_skip_v = g_fault.skip_v;

    static unsigned char done_attn[kMaxDevices];
    cudaError_t e;
    if ((e = opt_in_smem(tc::attention_kernel<false>, tc::attn::SMEM, done_attn)) != cudaSuccess) return HYB_ERR_CUDA;
    const uint64_t row_bytes = (uint64_t)H * D * 2;
    CUtensorMap tq, tk, tv, tout;
    if (!map3d(&tq, q, (uint64_t)H * D, T, B, row_bytes, row_bytes * T) ||
        !map3d(&tk, k_cache, (uint64_t)H * D, a.T_kv, B, row_bytes, row_bytes * cache_tokens) ||
        !map3d(&tv, v_cache, (uint64_t)H * D, a.T_kv, B, row_bytes, row_bytes * cache_tokens) ||
        !map3d(&tout, out, (uint64_t)H * D, T, B, row_bytes, row_bytes * T))
        return HYB_ERR_CUDA;
    cudaLaunchConfig_t acfg = {};
    acfg.gridDim = dim3(attn_tiles(T), H, B);
    acfg.blockDim = dim3(tc::attn::kThreads, 1, 1);
    acfg.dynamicSmemBytes = tc::attn::SMEM;
    acfg.stream = st;
    cudaError_t le = cudaSuccess;
    // tq stands in for the unused W map
    e = timed(K_ATTN, st, [&] { le = cudaLaunchKernelEx(&acfg, tc::attention_kernel<false>, a, tq, tk, tv, tq, tout); });
    if (e != cudaSuccess || le != cudaSuccess) return HYB_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? HYB_OK : HYB_ERR_CUDA;
}

}  // namespace

extern "C" {

hyb_status hyb_kvcache_attn_forward(const hyb_attn_desc* desc, const void* q, const void* k, const void* v,
                                    void* k_cache, void* v_cache, int cache_tokens, int cached_tokens, void* out,
                                    void* workspace, size_t workspace_bytes, void* stream) {
    return kvcache_impl(desc, q, k, v, k_cache, v_cache, cache_tokens, cached_tokens, out, workspace,
                        workspace_bytes, stream);
}

size_t hyb_attn_workspace_bytes(const hyb_attn_desc* desc) {
    Plan p;
    return make_plan(desc, &p) == HYB_OK ? p.total : 0;
}

hyb_status hyb_attn_forward(const hyb_attn_desc* desc, const void* q, const void* k, const void* v,
                            const void* phi_q, const void* phi_k, const void* phi_v,
                            const float* gate_logits, const float* beta_logits, float* state,
                            int clean_pass, void* out, void* workspace, size_t workspace_bytes,
                            void* stream) {
    if (!out) return HYB_ERR_INVALID;
    return forward_impl(desc, q, k, v, phi_q, phi_k, phi_v, gate_logits, beta_logits, state,
                        clean_pass, out, nullptr, nullptr, workspace, workspace_bytes, stream);
}

hyb_status hyb_attn_forward_branches(const hyb_attn_desc* desc, const void* q, const void* k,
                                     const void* v, const void* phi_q, const void* phi_k,
                                     const void* phi_v, const float* gate_logits,
                                     const float* beta_logits, float* state, int clean_pass,
                                     void* out, float* out_intra, float* out_inter,
                                     void* workspace, size_t workspace_bytes, void* stream) {
    if (!out_intra || !out_inter) return HYB_ERR_INVALID;
    return forward_impl(desc, q, k, v, phi_q, phi_k, phi_v, gate_logits, beta_logits, state,
                        clean_pass, out, out_intra, out_inter, workspace, workspace_bytes, stream);
}

hyb_status hyb_attn_forward_mixed(const hyb_attn_desc* desc, const void* q, const void* k, const void* v,
                                  const void* phi_q, const void* phi_k, const void* phi_v,
                                  const float* gate_logits, const float* beta_logits, float* state,
                                  int clean_pass, const float* mix, void* out, void* workspace,
                                  size_t workspace_bytes, void* stream) {
    if (!mix || !out) return HYB_ERR_INVALID;
    return forward_impl(desc, q, k, v, phi_q, phi_k, phi_v, gate_logits, beta_logits, state, clean_pass, out,
                        nullptr, nullptr, workspace, workspace_bytes, stream, mix);
}

hyb_status hyb_attn_forward_next(const hyb_attn_desc* desc, const void* q, const void* k, const void* v,
                                 const void* phi_q, const void* phi_k, const void* phi_v,
                                 const float* gate_logits, const float* beta_logits, float* state,
                                 int clean_pass, void* out, void* workspace, size_t workspace_bytes,
                                 void* stream) {
    if (!out) return HYB_ERR_INVALID;
    ChainRec prev;
    const bool had = chain_find(workspace, &prev);
    LayerArgs a;
    Plan p;
    hyb_status s = pass_args(desc, q, k, v, phi_q, phi_k, phi_v, gate_logits, beta_logits, state, clean_pass,
                             out, nullptr, nullptr, workspace, workspace_bytes, nullptr, &a, &p);
    if (s != HYB_OK) return s;
    if (!p.bf16) return launch_pass(a, p, clean_pass, stream);  // the fp32 path keeps no chain
    cudaStream_t st = (cudaStream_t)stream;
    const bool cont = had && prev.state == state && prev.phi_q == phi_q && prev.stream == st &&
                      prev.B == desc->B && prev.H == desc->H && prev.T == desc->T && prev.dtype == desc->dtype &&
                      prev.d == desc->d_k && prev.sm_scale == desc->sm_scale && prev.l2_eps == desc->l2_eps;
    // W slots: the pass reads slot `cur` and its delta update writes the other,
    // which the attention kernel of this pass does not read
    char* ws = (char*)workspace;
    const size_t hh = (size_t)desc->B * desc->H * 128 * 128;
    __nv_bfloat16* slot[2] = {(__nv_bfloat16*)(ws + p.off_W), (__nv_bfloat16*)(ws + p.off_Sprev)};
    const int cur = cont ? prev.cur : 0;
    unsigned epoch = cont ? prev.epoch : 0;
    a.WT_hi = slot[cur];
    a.WT_lo = a.WT_hi + hh;
    if (clean_pass) {
        a.w_next = slot[1 - cur];
        a.chain_flags = (unsigned*)(ws + p.off_chain);
        a.chain_wait = epoch;
        a.chain_set = epoch = chain_next_epoch();
        a.chain_trigger = 1;
    }
    TcPass tp;
    cudaError_t e = tp.init(a);
    tp.a.q_per_cta = attn_q_per_cta(tp.a);
    // a continued chain has W of the present state in slot `cur` already (the
    // previous clean pass's update wrote it, or a prep before a query-only pass)
    if (e == cudaSuccess && !cont) e = tp.prep(st, true);
    if (e == cudaSuccess) e = tp.attn(st, true);
    if (e == cudaSuccess && clean_pass) e = tp.update(st, true);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return HYB_ERR_CUDA;
    ChainRec rec;
    rec.ws = workspace;
    rec.state = state;
    rec.phi_q = phi_q;
    rec.stream = st;
    rec.B = desc->B;
    rec.H = desc->H;
    rec.T = desc->T;
    rec.dtype = desc->dtype;
    rec.d = desc->d_k;
    rec.sm_scale = desc->sm_scale;
    rec.l2_eps = desc->l2_eps;
    rec.cur = clean_pass ? 1 - cur : cur;
    rec.epoch = epoch;
    chain_store(rec);
    return HYB_OK;
}

// ---- Token Radius Attention ------------------------------------------------------
static bool tra_params_ok(const hyb_attn_desc* d, const hyb_tra_params* p) {
    return p && p->grid_h > 0 && p->grid_w > 0 && p->grid_h < 32768 && p->grid_w < 32768 &&
           (long long)p->grid_h * p->grid_w == d->T && p->tile_h > 0 && p->tile_w > 0 && p->votes_min >= 1 &&
           p->tau > 0.f && isfinite(p->tau);
}

size_t hyb_tra_workspace_bytes(const hyb_attn_desc* desc) {
    Plan p;
    if (make_plan(desc, &p) != HYB_OK || !p.bf16) return 0;
    const size_t nkb = (desc->T + tra::kBlock - 1) / tra::kBlock;
    const size_t bh = (size_t)desc->B * desc->H;
    // block lists, their lengths, the schedule of the block-sparse grid, the mask
    // kernel's ticket
    return align_up(align_up(p.total, 256) + bh * nkb * nkb * sizeof(int), 256) +
           2 * align_up(bh * nkb * sizeof(int), 256) + 256;
}

hyb_status hyb_tra_forward(const hyb_attn_desc* desc, const hyb_tra_params* params, int warmup, const void* q,
                           const void* k, const void* v, const void* phi_q, const void* phi_k, const void* phi_v,
                           const float* gate_logits, const float* beta_logits, float* state, int clean_pass,
                           void* out, float* entropy, void* workspace, size_t workspace_bytes, void* stream) {
    if (!out || !entropy) return HYB_ERR_INVALID;
    Plan p;
    hyb_status s = make_plan(desc, &p);
    if (s != HYB_OK) return s;
    if (!p.bf16) return HYB_ERR_UNSUPPORTED;
    if (!tra_params_ok(desc, params) || (warmup != 0 && warmup != 1)) return HYB_ERR_INVALID;
    if (((uintptr_t)entropy & 15u) != 0) return HYB_ERR_ALIGN;
    const size_t need = hyb_tra_workspace_bytes(desc);
    if (!workspace || workspace_bytes < need) return HYB_ERR_WORKSPACE;
    LayerArgs a;
    s = pass_args(desc, q, k, v, phi_q, phi_k, phi_v, gate_logits, beta_logits, state, clean_pass, out, nullptr,
                  nullptr, workspace, workspace_bytes, nullptr, &a, &p);
    if (s != HYB_OK) return s;
    cudaStream_t st = (cudaStream_t)stream;
    const int nkb = (desc->T + tra::kBlock - 1) / tra::kBlock;
    int* list = (int*)((char*)workspace + align_up(p.total, 256));
    int* count = (int*)((char*)list + align_up((size_t)desc->B * desc->H * nkb * nkb * sizeof(int), 256));
    int* order = (int*)((char*)count + align_up((size_t)desc->B * desc->H * nkb * sizeof(int), 256));
    int* done = (int*)((char*)order + align_up((size_t)desc->B * desc->H * nkb * sizeof(int), 256));
    const size_t msm = tra::mask_smem_bytes(nkb);
    if (msm > 227u * 1024u) return HYB_ERR_UNSUPPORTED;
    if (warmup) {
        // dense pass; the attention kernel also writes every query's entropy, then
        // the block mask is built once from them (the later passes reuse it)
        static unsigned char done_mask[kMaxDevices];
        cudaError_t e = opt_in_smem(tra::mask_kernel, msm, done_mask);
        if (e != cudaSuccess) return HYB_ERR_CUDA;
        a.ent_out = entropy;
        if (launch_tc(a, clean_pass, st) != cudaSuccess) return HYB_ERR_CUDA;
        const tra::Params tp = {params->grid_h, params->grid_w, params->tile_h, params->tile_w, params->tau,
                                params->votes_min};
        tra::mask_kernel<<<dim3(nkb, desc->H, desc->B), tra::kMaskThreads, msm, st>>>(a, tp, entropy, list, count,
                                                                                       order, done);
        return cudaGetLastError() == cudaSuccess ? HYB_OK : HYB_ERR_CUDA;
    }
    // block-sparse pass: the attention kernel walks the kept key blocks of the
    // mask the last warm-up pass on this workspace built
    a.kv_list = list;
    a.kv_count = count;
    a.kv_stride = nkb;
    a.kv_order = order;
    return launch_tc(a, clean_pass, st) == cudaSuccess ? HYB_OK : HYB_ERR_CUDA;
}

size_t hyb_attn_frames_workspace_bytes(const hyb_attn_desc* desc, int n_frames) {
    Plan p;
    if (n_frames < 1 || n_frames > kMaxFrames || make_plan(desc, &p) != HYB_OK) return 0;
    return frames_total(desc, p, n_frames);
}

hyb_status hyb_attn_forward_frames(const hyb_attn_desc* desc, int n_frames, const void* q, const void* k,
                                   const void* v, const void* phi_q, const void* phi_k, const void* phi_v,
                                   const float* gate_logits, const float* beta_logits, float* state, void* out,
                                   void* workspace, size_t workspace_bytes, void* stream) {
    Plan p;
    hyb_status s = make_plan(desc, &p);
    if (s != HYB_OK) return s;
    if (n_frames < 1 || n_frames > kMaxFrames) return HYB_ERR_INVALID;
    if (!q || !k || !v || !out || !gate_logits || !beta_logits) return HYB_ERR_INVALID;
    if (!workspace || workspace_bytes < frames_total(desc, p, n_frames)) return HYB_ERR_WORKSPACE;
    const size_t esz = p.bf16 ? 2 : 4;
    const size_t fe = (size_t)desc->B * desc->T * desc->H * p.D * esz;  // bytes of q (k, v, out) per frame
    const size_t fg = (size_t)desc->B * desc->H * desc->T;              // gate logits per frame
    LayerArgs* args = new (std::nothrow) LayerArgs[n_frames];
    if (!args) return HYB_ERR_INVALID;
    // every frame's arguments are checked before anything is enqueued
    for (int n = 0; n < n_frames && s == HYB_OK; ++n)
        s = pass_args(desc, (const char*)q + n * fe, (const char*)k + n * fe, (const char*)v + n * fe, phi_q, phi_k,
                      phi_v, gate_logits + n * fg, beta_logits + n * fg, state, 1, (char*)out + n * fe, nullptr,
                      nullptr, workspace, workspace_bytes, nullptr, &args[n], &p);
    if (s != HYB_OK) {
        delete[] args;
        return s;
    }
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = cudaSuccess;
    if (!p.bf16) {
        // fp32 path: the frames one after another on the caller's stream
        for (int n = 0; n < n_frames && e == cudaSuccess; ++n) e = launch_simt<32, float>(args[n], 1, st);
        delete[] args;
        return e == cudaSuccess ? HYB_OK : HYB_ERR_CUDA;
    }
    // bf16: the state chain (W_N = phi_q^T S_{N-1}, then S_N) on one stream, the
    // attention kernels on two others, frame after frame in turn; attention of
    // frame N waits only for W_N, so the attention kernels of consecutive frames
    // share the SMs (the next frame's first wave starts beside this frame's
    // second) instead of each ending on a partial wave.  Each frame's W has its
    // own slot.
    FrameRes* r = nullptr;
    if ((e = frame_resources(n_frames, &r)) != cudaSuccess) {
        delete[] args;
        return HYB_ERR_CUDA;
    }
    const size_t wslot = align_up(frames_w_bytes(desc, p), 256);
    char* slots = (char*)workspace + align_up(p.total, 256);
    const size_t hh = (size_t)desc->B * desc->H * p.D * p.D;
    TcPass* tp = new (std::nothrow) TcPass[n_frames];
    if (!tp) {
        delete[] args;
        return HYB_ERR_INVALID;
    }
    unsigned prev_epoch = 0;
    for (int n = 0; n < n_frames && e == cudaSuccess; ++n) {
        args[n].WT_hi = (__nv_bfloat16*)(slots + n * wslot);
        args[n].WT_lo = args[n].WT_hi + hh;
        // the update of frame n also writes W of frame n + 1 (what prep would
        // compute from S_n), so the chain is one kernel per frame
        args[n].w_next = n + 1 < n_frames ? (__nv_bfloat16*)(slots + (n + 1) * wslot) : nullptr;
        // consecutive updates overlap: update n + 1 starts (PDL) once every CTA
        // of update n has finished its key tiles, walks its own, and waits for
        // update n's flags before it reads S_n (at most two updates hold SMs)
        args[n].chain_flags = (unsigned*)((char*)workspace + p.off_chain);
        args[n].chain_wait = prev_epoch;
        args[n].chain_set = prev_epoch = chain_next_epoch();
        args[n].chain_trigger = 2;
        e = tp[n].init(args[n]);
    }
    if (e == cudaSuccess) e = cudaEventRecord(r->fork, st);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(r->chain, r->fork, 0);
    for (int i = 0; i < kAttStreams && e == cudaSuccess; ++i) e = cudaStreamWaitEvent(r->att[i], r->fork, 0);
    if (e == cudaSuccess) e = tp[0].prep(r->chain, false);
    if (e == cudaSuccess) e = cudaEventRecord(r->w[0], r->chain);
    for (int n = 0; n < n_frames && e == cudaSuccess; ++n) {
        if ((e = tp[n].update(r->chain, n > 0)) != cudaSuccess) break;
        if (n + 1 < n_frames && (e = cudaEventRecord(r->w[n + 1], r->chain)) != cudaSuccess) break;
        cudaStream_t att = r->att[n % kAttStreams];
        if ((e = cudaStreamWaitEvent(att, r->w[n], 0)) != cudaSuccess) break;
        e = tp[n].attn(att, false);
    }
    // join: the caller's stream continues after every frame's kernels
    if (e == cudaSuccess) e = cudaEventRecord(r->join_chain, r->chain);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(st, r->join_chain, 0);
    for (int i = 0; i < kAttStreams && e == cudaSuccess; ++i) {
        if ((e = cudaEventRecord(r->join_att[i], r->att[i])) == cudaSuccess) e = cudaStreamWaitEvent(st, r->join_att[i], 0);
    }
    delete[] tp;
    delete[] args;
    if (e == cudaSuccess) e = cudaGetLastError();
    return e == cudaSuccess ? HYB_OK : HYB_ERR_CUDA;
}

size_t hyb_attn_token_level_workspace_bytes(const hyb_attn_desc* desc) {
    Plan p;
    if (make_plan(desc, &p) != HYB_OK) return 0;
    return tok_plan(desc, p).total;
}

hyb_status hyb_attn_forward_token_level(const hyb_attn_desc* desc, const void* q, const void* k, const void* v,
                                        const void* phi_q, const void* phi_k, const void* phi_v,
                                        const float* gate_logits, const float* beta_logits, float* state,
                                        int clean_pass, void* out, void* workspace, size_t workspace_bytes,
                                        void* stream) {
    if (!out) return HYB_ERR_INVALID;
    Plan p;
    hyb_status s = make_plan(desc, &p);
    if (s != HYB_OK) return s;
    const TokPlan tp = tok_plan(desc, p);
    if (workspace && workspace_bytes < tp.total) return HYB_ERR_WORKSPACE;
    LayerArgs a;
    s = pass_args(desc, q, k, v, phi_q, phi_k, phi_v, gate_logits, beta_logits, state, clean_pass, out, nullptr,
                  nullptr, workspace, workspace_bytes, nullptr, &a, &p);
    if (s != HYB_OK) return s;
    // a query-only pass reads the frame-start state with every token: it is the
    // frame-level pass
    if (!clean_pass) return launch_pass(a, p, 0, stream);
    cudaError_t e;
    if (p.bf16)
        e = launch_token_level<128, __nv_bfloat16>(a, tp, (char*)workspace, (cudaStream_t)stream);
    else
        e = launch_token_level<32, float>(a, tp, (char*)workspace, (cudaStream_t)stream);
    return e == cudaSuccess ? HYB_OK : HYB_ERR_CUDA;
}

hyb_status hyb_attn_get_device_status(const void* workspace, void* stream) {
    if (!workspace) return HYB_ERR_INVALID;
    if (!aligned16(workspace)) return HYB_ERR_ALIGN;
    cudaStream_t st = (cudaStream_t)stream;
    if (cudaStreamSynchronize(st) != cudaSuccess) return HYB_ERR_CUDA;
    unsigned flags = 0;
    if (cudaMemcpy(&flags, workspace, sizeof(flags), cudaMemcpyDeviceToHost) != cudaSuccess)
        return HYB_ERR_CUDA;
    if (flags && cudaMemset((void*)workspace, 0, sizeof(flags)) != cudaSuccess) return HYB_ERR_CUDA;
    if (flags & FLAG_INTERNAL) return HYB_ERR_CUDA;
    if (flags & FLAG_TIMEOUT) return HYB_ERR_TIMEOUT;
    if (flags & FLAG_NONFINITE) return HYB_WARN_NONFINITE;
    return HYB_OK;
}

hyb_status hyb_attn_set_fault_test(int skip_v_loads, unsigned wait_limit_us) {
    if (skip_v_loads != 0 && skip_v_loads != 1) return HYB_ERR_INVALID;
    if (wait_limit_us > 10u * 1000u * 1000u) return HYB_ERR_INVALID;
    g_fault.skip_v = skip_v_loads;
    g_fault.wait_ns = wait_limit_us ? (unsigned long long)wait_limit_us * 1000ull : 2000000000ull;
    return HYB_OK;
}

hyb_status hyb_attn_timing_begin(int max_launches) {
    if (g_timing.on || max_launches <= 0 || max_launches > (1 << 20)) return HYB_ERR_INVALID;
    g_timing.ev = new (std::nothrow) cudaEvent_t[2 * (size_t)max_launches];
    g_timing.kind = new (std::nothrow) int[max_launches];
    if (!g_timing.ev || !g_timing.kind) {
        delete[] g_timing.ev;
        delete[] g_timing.kind;
        g_timing.ev = nullptr;
        g_timing.kind = nullptr;
        return HYB_ERR_INVALID;
    }
    int made = 0;
    for (; made < 2 * max_launches; ++made)
        if (cudaEventCreate(&g_timing.ev[made]) != cudaSuccess) break;
    if (made < 2 * max_launches) {
        for (int i = 0; i < made; ++i) cudaEventDestroy(g_timing.ev[i]);
        delete[] g_timing.ev;
        delete[] g_timing.kind;
        g_timing.ev = nullptr;
        g_timing.kind = nullptr;
        return HYB_ERR_CUDA;
    }
    g_timing.cap = max_launches;
    g_timing.used = 0;
    g_timing.dropped = 0;
    g_timing.on = true;
    return HYB_OK;
}

hyb_status hyb_attn_timing_end(hyb_attn_timing* out) {
    if (!g_timing.on) return HYB_ERR_INVALID;
    hyb_status st = HYB_OK;
    hyb_attn_timing t;
    memset(&t, 0, sizeof(t));
    for (int i = 0; i < g_timing.used; ++i) {
        float ms = 0.f;
        if (cudaEventSynchronize(g_timing.ev[2 * i + 1]) != cudaSuccess ||
            cudaEventElapsedTime(&ms, g_timing.ev[2 * i], g_timing.ev[2 * i + 1]) != cudaSuccess) {
            st = HYB_ERR_CUDA;
            continue;
        }
        t.launches[g_timing.kind[i]] += 1;
        t.total_ms[g_timing.kind[i]] += ms;
    }
    t.dropped = g_timing.dropped;
    for (int i = 0; i < 2 * g_timing.cap; ++i) cudaEventDestroy(g_timing.ev[i]);
    delete[] g_timing.ev;
    delete[] g_timing.kind;
    g_timing = Timing();
    if (out) *out = t;
    return st;
}

const char* hyb_attn_kernel_name(int kernel) {
    static const char* names[HYB_NUM_KERNELS] = {"prep", "intra_frame_attention", "delta_update",
                                                 "delta_update_apply", "token_chunk_prep", "token_chain",
                                                 "token_reads"};
    return (kernel >= 0 && kernel < HYB_NUM_KERNELS) ? names[kernel] : nullptr;
}

const char* hyb_attn_status_string(hyb_status s) {
    switch (s) {
        case HYB_OK: return "HYB_OK";
        case HYB_WARN_NONFINITE: return "HYB_WARN_NONFINITE: a state update produced inf/NaN";
        case HYB_ERR_INVALID: return "HYB_ERR_INVALID: invalid argument";
        case HYB_ERR_UNSUPPORTED: return "HYB_ERR_UNSUPPORTED: unsupported dtype/shape";
        case HYB_ERR_ALIGN: return "HYB_ERR_ALIGN: pointer not 16-byte aligned";
        case HYB_ERR_WORKSPACE: return "HYB_ERR_WORKSPACE: workspace missing or too small";
        case HYB_ERR_CUDA: return "HYB_ERR_CUDA: CUDA call or launch failed";
        case HYB_ERR_TIMEOUT: return "HYB_ERR_TIMEOUT: a bounded device wait gave up";
    }
    return "unknown hyb_status";
}

}  // extern "C"

// ---- zero-allocation variant --------------------------------------------------
// Scratch for hyb_attn_forward_noalloc: a fixed array in the library's own
// device memory, so that callers which may not allocate (graph capture in a
// strict mode, allocator callbacks, fixed-budget serving loops) can run a pass
// without a workspace.  Every GPU that loads the library holds it until exit.
static __device__ __align__(256) unsigned char g_noalloc_scratch[HYB_NOALLOC_SCRATCH_BYTES];

namespace {
// Device address of g_noalloc_scratch per device, looked up once with that
// device current.  In host code the array's name is only a host-side stand-in.
void* g_noalloc_ptr[kMaxDevices];

void* noalloc_scratch(cudaError_t* err) {
    int dev = 0;
    *err = cudaGetDevice(&dev);
    if (*err != cudaSuccess) return nullptr;
    if (dev < 0 || dev >= kMaxDevices) {
        *err = cudaErrorInvalidDevice;
        return nullptr;
    }
    if (!g_noalloc_ptr[dev]) {
        void* ptr = nullptr;
        *err = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (*err != cudaSuccess) return nullptr;
        g_noalloc_ptr[dev] = ptr;
    }
    return g_noalloc_ptr[dev];
}
}  // namespace

extern "C" hyb_status hyb_attn_forward_noalloc(const hyb_attn_desc* desc, const void* q, const void* k,
                                               const void* v, const void* phi_q, const void* phi_k,
                                               const void* phi_v, const float* gate_logits,
                                               const float* beta_logits, float* state, int clean_pass,
                                               void* out, void* stream) {
    if (!out) return HYB_ERR_INVALID;
    Plan p;
    hyb_status s = make_plan(desc, &p);
    if (s != HYB_OK) return s;
    if (p.total > (size_t)HYB_NOALLOC_SCRATCH_BYTES) return HYB_ERR_WORKSPACE;
    // every argument is checked before any CUDA call (with a stand-in for the
    // scratch address, which is looked up only afterwards)
    LayerArgs a;
    s = pass_args(desc, q, k, v, phi_q, phi_k, phi_v, gate_logits, beta_logits, state, clean_pass, out, nullptr,
                  nullptr, (void*)(uintptr_t)256, HYB_NOALLOC_SCRATCH_BYTES, nullptr, &a, &p);
    if (s != HYB_OK) return s;
    cudaError_t e;
    void* scratch = noalloc_scratch(&e);
    if (!scratch) return HYB_ERR_CUDA;
    s = pass_args(desc, q, k, v, phi_q, phi_k, phi_v, gate_logits, beta_logits, state, clean_pass, out, nullptr,
                  nullptr, scratch, HYB_NOALLOC_SCRATCH_BYTES, nullptr, &a, &p);
    if (s != HYB_OK) return s;
    // the status word accumulates flags: start every call from zero
    if (cudaMemsetAsync(scratch, 0, sizeof(unsigned), (cudaStream_t)stream) != cudaSuccess)
        return HYB_ERR_CUDA;
    return launch_pass(a, p, clean_pass, stream);
}

extern "C" hyb_status hyb_attn_noalloc_device_status(void* stream) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return HYB_ERR_CUDA;
    // the scratch address is known once a call on this device has looked it up
    if (!g_noalloc_ptr[dev]) return HYB_OK;
    return hyb_attn_get_device_status(g_noalloc_ptr[dev], stream);
}
