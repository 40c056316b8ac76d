// tra.cuh -- Token Radius Attention on the intra-frame branch: the block mask.
//
// Source: "Technical summary: Token Radius Attention", gist.science/ar/paper/
// 2608.02504, §2: a dense warm-up pass gives each query its attention entropy H
// (written by the attention kernel's warm-up variant); the entropy maps to a
// budget of keys, the budget to a spatial radius around the query on the
// frame's patch grid; over a tile-major token order the token-radius masks are
// turned into a block-sparse mask by distance tests and token voting, and the
// attention then walks only the kept key blocks.
//
// Readings (also in the API header): budget k = clamp(tau exp(H), 1, T) keys,
// radius r = sqrt(k / pi) patches (the temporal decay exp(-gamma delta) is 1 on
// the current frame, the only one the intra-frame branch attends to); tokens
// are in tile-major order (tiles of tile_h x tile_w patches row-major over the
// grid, patches row-major inside a tile, edge tiles cut); a query votes for a key
// block when some key of the block lies within its radius (Euclidean distance on
// patch coordinates); a key block is kept for a query block with at least
// votes_min votes, and always for itself.
#pragma once

#include "common.cuh"

namespace hyb {
namespace tra {

constexpr int kBlock = 128;  // tokens per query / key block (the attention kernel's tile)

struct Params {
    int grid_h, grid_w, tile_h, tile_w;
    float tau;
    int votes_min;
};

// Patch (row, col) of token t in tile-major order.
__device__ __forceinline__ void tile_major_pos(int t, const Params& p, int* r, int* c) {
    const int tr = t / (p.tile_h * p.grid_w);          // tile row (all earlier ones are full height)
    const int rem = t - tr * p.tile_h * p.grid_w;
    const int hr = min(p.tile_h, p.grid_h - tr * p.tile_h);
    const int tc = rem / (hr * p.tile_w);              // tile within the row (earlier ones full width)
    const int rem2 = rem - tc * hr * p.tile_w;
    const int wc = min(p.tile_w, p.grid_w - tc * p.tile_w);
    *r = tr * p.tile_h + rem2 / wc;
    *c = tc * p.tile_w + rem2 % wc;
}

// Squared radius of a query with entropy H, in fp32: clamp(tau exp(H), 1, T) / pi.
__device__ __forceinline__ float radius2(float H, float tau, int T) {
    return fminf(fmaxf(tau * expf(H), 1.0f), (float)T) * 0.31830988618379067f;
}

// Shared memory: key-block boxes [nkb] int4, run counts [nkb] ints, votes [nkb]
// ints, runs [nkb * kBlock] int2.
__host__ __device__ inline size_t mask_smem_bytes(int nkb) {
    return (size_t)nkb * (sizeof(int4) + 2 * sizeof(int) + kBlock * sizeof(int2));
}

// One CTA of kMaskThreads per (query block, head, batch): four warps per 32
// queries of the block, each of the four taking every fourth key block (the
// tests are short and latency-bound, so more warps per SM, not fewer, hide it).
// Writes the ascending list of kept key blocks of the query block at
// list[(bh * nkb + qb) * nkb] and its length at count[bh * nkb + qb].  The CTA
// that finishes last (an atomic ticket on *done, which it resets) then orders
// the rows (bh * nkb + qb) by list length, longest first, into order[]: a
// counting sort (rows of equal length in any order, as each row's result does
// not depend on when it runs).  The block-sparse attention grid takes its rows
// in this order: CTAs are dispatched in grid order, so its second wave holds
// the shortest lists and ends with the first.
//
// A key block is described by its bounding box and by its runs: maximal
// stretches of consecutive tokens on one patch row with consecutive columns
// (a tile's row, or the part of it inside the block).  The distance from a
// query to a run is exact (row offset and the column gap to the run's span),
// so a query's vote needs one test per run instead of one per key; when the
// block fills its box (a whole tile, or rows of one), the box test alone is
// exact.  Decisions are those of the per-key test: the same integer squared
// distances against the same fp32 squared radius.
constexpr int kMaskThreads = 512;
constexpr int kKbGroups = kMaskThreads / kBlock;  // warps that share a query's key blocks
__global__ void __launch_bounds__(kMaskThreads) mask_kernel(LayerArgs a, Params p, const float* __restrict__ ent,
                                                      int* __restrict__ list, int* __restrict__ count,
                                                      int* __restrict__ order, int* __restrict__ done) {
    extern __shared__ __align__(16) unsigned char msm[];
    const int T = a.T;
    const int nkb = (T + kBlock - 1) / kBlock;
    int4* box = reinterpret_cast<int4*>(msm);                                 // (r0, r1, c0, c1)
    int2* run = reinterpret_cast<int2*>(msm + (size_t)nkb * sizeof(int4));    // ((r << 16) | c0, c1)
    int* nrun = reinterpret_cast<int*>(run + (size_t)nkb * kBlock);           // runs; -runs if the box is full
    int* votes = nrun + nkb;
    const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t bh = (size_t)b * a.H + h;
    for (int kb = tid; kb < nkb; kb += kMaskThreads) votes[kb] = 0;
    // runs and bounding box of each key block (a warp per block)
    for (int kb = warp; kb < nkb; kb += kMaskThreads / 32) {
        const int ntok = min(kBlock, T - kb * kBlock);
        int r0 = 1 << 30, r1 = -1, c0 = 1 << 30, c1 = -1;
        int nstart = 0, nend = 0;
        for (int base = 0; base < ntok; base += 32) {
            const int i = base + lane, j = kb * kBlock + i;
            const bool valid = i < ntok;
            int r = 0, c = 0, rp = -1, cp = -2, rn = -1, cn = -2;
            if (valid) {
                tile_major_pos(j, p, &r, &c);
                if (i > 0) tile_major_pos(j - 1, p, &rp, &cp);
                if (i + 1 < ntok) tile_major_pos(j + 1, p, &rn, &cn);
                r0 = min(r0, r);
                r1 = max(r1, r);
                c0 = min(c0, c);
                c1 = max(c1, c);
            }
            const bool start = valid && !(rp == r && cp + 1 == c);
            const bool end = valid && !(rn == r && cn == c + 1);
            const unsigned ms = __ballot_sync(0xffffffffu, start), me = __ballot_sync(0xffffffffu, end);
            const unsigned below = (1u << lane) - 1u;
            if (start) run[kb * kBlock + nstart + __popc(ms & below)].x = (r << 16) | c;
            if (end) run[kb * kBlock + nend + __popc(me & below)].y = c;
            nstart += __popc(ms);
            nend += __popc(me);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            r0 = min(r0, __shfl_xor_sync(0xffffffffu, r0, o));
            r1 = max(r1, __shfl_xor_sync(0xffffffffu, r1, o));
            c0 = min(c0, __shfl_xor_sync(0xffffffffu, c0, o));
            c1 = max(c1, __shfl_xor_sync(0xffffffffu, c1, o));
        }
        if (lane == 0) {
            box[kb] = make_int4(r0, r1, c0, c1);
            const bool full = (r1 - r0 + 1) * (c1 - c0 + 1) == ntok;
            nrun[kb] = full ? -nstart : nstart;
        }
    }
    __syncthreads();
    const int t = qb * kBlock + (warp % (kBlock / 32)) * 32 + lane;   // this thread's query
    const int kb0 = warp / (kBlock / 32);                               // its first key block
    const bool valid = t < T;
    const float r2 = valid ? radius2(ent[bh * T + t], p.tau, T) : -1.0f;
    int rq = 0, cq = 0;
    if (valid) tile_major_pos(t, p, &rq, &cq);
    for (int kb = kb0; kb < nkb; kb += kKbGroups) {
        const int4 bb = box[kb];
        const int dy = max(0, max(bb.x - rq, rq - bb.y)), dx = max(0, max(bb.z - cq, cq - bb.w));
        bool hit = false;
        if (valid && (float)(dy * dy + dx * dx) <= r2) {
            const int nr = nrun[kb];
            if (nr < 0) {
                hit = true;  // the block fills its box: the nearest point of the box is a key
            } else {
                for (int u = 0; u < nr; ++u) {
                    const int2 ru = run[kb * kBlock + u];
                    const int ry = (ru.x >> 16) - rq;
                    const int rx = max(0, max((ru.x & 0xffff) - cq, cq - ru.y));
                    if ((float)(ry * ry + rx * rx) <= r2) {
                        hit = true;
                        break;
                    }
                }
            }
        }
        const int nv = __popc(__ballot_sync(0xffffffffu, hit));
        if (lane == 0 && nv) atomicAdd(&votes[kb], nv);
    }
    __syncthreads();
    volatile int* last = nrun;  // (free now) the ticket's verdict for the whole CTA
    if (tid == 0) {
        const size_t row = bh * nkb + qb;
        int cnt = 0;
        for (int kb = 0; kb < nkb; ++kb)
            if (votes[kb] >= p.votes_min || kb == qb) list[row * nkb + cnt++] = kb;
        count[row] = cnt;
        __threadfence();
        const int ctas = gridDim.x * gridDim.y * gridDim.z;
        const int ticket = atomicAdd(done, 1);
        *last = ticket == ctas - 1;
        if (ticket == ctas - 1) {
            *done = 0;  // for the next mask
            __threadfence();
        }
    }
    __syncthreads();
    if (!*last) return;
    // the last CTA: counting sort of the rows by list length (every CTA's count
    // is visible: each wrote it before its ticket)
    const int rows = gridDim.x * gridDim.y * gridDim.z;
    int* slot = reinterpret_cast<int*>(box);  // [nkb + 1]: rows of each length, then first positions
    for (int c = tid; c <= nkb; c += kMaskThreads) slot[c] = 0;
    __syncthreads();
    for (int i = tid; i < rows; i += kMaskThreads) atomicAdd(&slot[min(max(__ldcg(count + i), 0), nkb)], 1);
    __syncthreads();
    if (tid == 0) {
        int pos = 0;
        for (int c = nkb; c >= 0; --c) {
            const int k = slot[c];
            slot[c] = pos;
            pos += k;
        }
    }
    __syncthreads();
    for (int i = tid; i < rows; i += kMaskThreads)
        order[atomicAdd(&slot[min(max(__ldcg(count + i), 0), nkb)], 1)] = i;
}

}  // namespace tra
}  // namespace hyb
