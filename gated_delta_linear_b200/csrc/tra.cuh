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

// Shared memory: votes [nkb] ints, key-block boxes [nkb] int4, key positions [nkb * kBlock] ints.
__host__ __device__ inline size_t mask_smem_bytes(int nkb) {
    return (size_t)nkb * (sizeof(int) + sizeof(int4) + kBlock * sizeof(int));
}

// One CTA per (query block, head, batch), a thread per query of the block.
// Writes the ascending list of kept key blocks of the query block at
// list[(bh * nkb + qb) * nkb] and its length at count[bh * nkb + qb].
__global__ void __launch_bounds__(kBlock) mask_kernel(LayerArgs a, Params p, const float* __restrict__ ent,
                                                      int* __restrict__ list, int* __restrict__ count) {
    extern __shared__ __align__(16) unsigned char msm[];
    const int T = a.T;
    const int nkb = (T + kBlock - 1) / kBlock;
    int4* box = reinterpret_cast<int4*>(msm);                                 // (r0, r1, c0, c1)
    int* kpos = reinterpret_cast<int*>(msm + (size_t)nkb * sizeof(int4));     // (r << 16) | c
    int* votes = kpos + (size_t)nkb * kBlock;
    const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t bh = (size_t)b * a.H + h;
    for (int j = tid; j < nkb * kBlock; j += kBlock) {
        int r = 0, c = 0;
        if (j < T) tile_major_pos(j, p, &r, &c);
        kpos[j] = (r << 16) | c;
    }
    for (int kb = tid; kb < nkb; kb += kBlock) votes[kb] = 0;
    __syncthreads();
    // bounding box of each key block's patches (a warp per block)
    for (int kb = warp; kb < nkb; kb += kBlock / 32) {
        int r0 = 1 << 30, r1 = -1, c0 = 1 << 30, c1 = -1;
        for (int jj = lane; jj < kBlock; jj += 32) {
            const int j = kb * kBlock + jj;
            if (j >= T) break;
            const int r = kpos[j] >> 16, c = kpos[j] & 0xffff;
            r0 = min(r0, r);
            r1 = max(r1, r);
            c0 = min(c0, c);
            c1 = max(c1, c);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            r0 = min(r0, __shfl_xor_sync(0xffffffffu, r0, o));
            r1 = max(r1, __shfl_xor_sync(0xffffffffu, r1, o));
            c0 = min(c0, __shfl_xor_sync(0xffffffffu, c0, o));
            c1 = max(c1, __shfl_xor_sync(0xffffffffu, c1, o));
        }
        if (lane == 0) box[kb] = make_int4(r0, r1, c0, c1);
    }
    __syncthreads();
    const int t = qb * kBlock + tid;
    const bool valid = t < T;
    const float r2 = valid ? radius2(ent[bh * T + t], p.tau, T) : -1.0f;
    const int rq = valid ? kpos[t] >> 16 : 0, cq = valid ? kpos[t] & 0xffff : 0;
    for (int kb = 0; kb < nkb; ++kb) {
        const int4 bb = box[kb];
        const int dy = max(0, max(bb.x - rq, rq - bb.y)), dx = max(0, max(bb.z - cq, cq - bb.w));
        bool hit = false;
        if (valid && (float)(dy * dy + dx * dx) <= r2) {
            for (int jj = 0; jj < kBlock; ++jj) {
                const int j = kb * kBlock + jj;
                if (j >= T) break;
                const int ry = (kpos[j] >> 16) - rq, rx = (kpos[j] & 0xffff) - cq;
                if ((float)(ry * ry + rx * rx) <= r2) {
                    hit = true;
                    break;
                }
            }
        }
        const int nv = __popc(__ballot_sync(0xffffffffu, hit));
        if (lane == 0 && nv) atomicAdd(&votes[kb], nv);
    }
    __syncthreads();
    if (tid == 0) {
        const size_t row = bh * nkb + qb;
        int cnt = 0;
        for (int kb = 0; kb < nkb; ++kb)
            if (votes[kb] >= p.votes_min || kb == qb) list[row * nkb + cnt++] = kb;
        count[row] = cnt;
    }
}

}  // namespace tra
}  // namespace hyb
