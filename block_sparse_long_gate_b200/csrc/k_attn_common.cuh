// k_attn_common.cuh - work decomposition shared by the attention kernels.
//
// Work items (one 128-row tile each), in launch order:
//   [0, P)           past tiles: up to 128 consecutive entries of one query list
//                    l = (b, hk, j); all keys of block j, no mask; result is a
//                    partial (O normalised by its own sum, lse) stored in the
//                    entry's slot.
//   [Pmax, Pmax + D) own-block ("diagonal") tiles: up to 128 consecutive tokens
//                    of one query head inside one block c; keys c*bs .. t with
//                    the causal mask; the partial goes to out / lse and is merged
//                    later. In dense mode the key range starts at 0 and the
//                    normalised result is final.
// P (the real number of past tiles) is only known on the device; items in
// [P, Pmax) exit at once.
#pragma once
#include "common.cuh"
#include "k_invert.cuh"

struct AttnParams {
    const uint16_t* q;
    const uint16_t* k;
    const uint16_t* v;
    int64_t N;
    int B, Hq, Hkv, G, bs, topk, kp;
    int64_t nblk, nch;
    // past tiles
    const uint64_t* entries;
    const int64_t* segoff;      // list l spans entries [segoff[l*nch], segoff[(l+1)*nch])
    const int64_t* tile_start;  // past tile prefix per list, tile_start[L] = P
    int64_t L, Pmax;
    uint16_t* opart;  // bf16 [B, Hq, N, kp, d]
    float* lpart;     // fp32 [B, Hq, N, kp]
    // diagonal / dense tiles
    int64_t D;
    int64_t mb, ml, per_bh;  // tiles per full block, in the last block, per (b, hq)
    int dense;               // 1: dense causal attention, key range starts at 0
    uint16_t* out;           // bf16 [B, N, Hq, d]
    float* lse;              // fp32 [B, Hq, N]
    float scale_log2;        // log2(e) / sqrt(d)
};

// Largest l with tile_start[l] <= p (lists without tiles are skipped).
__device__ __forceinline__ int64_t find_list(const int64_t* __restrict__ ts, int64_t L, int64_t p) {
    int64_t lo = 0, hi = L;  // invariant: ts[lo] <= p < ts[hi]
    while (hi - lo > 1) {
        int64_t mid = (lo + hi) >> 1;
        if (ts[mid] <= p) lo = mid;
        else hi = mid;
    }
    return lo;
}

struct TileInfo {
    int kind;         // 0 = past, 1 = diagonal / dense, -1 = nothing to do
    int b, hk;
    int64_t j;        // key block of a past tile
    int64_t e0, ne;   // past: first entry and count
    int hq;           // diagonal: query head
    int64_t t0, nt;   // diagonal: first token and count
    int64_t klo;      // first key
    int64_t khi;      // one past the last key any row of the tile reads
};

__device__ __forceinline__ TileInfo decode_tile(const AttnParams& a, int64_t item) {
    TileInfo ti;
    ti.kind = -1;
    if (item < a.Pmax) {
        const int64_t P = a.tile_start[a.L];
        if (item >= P) return ti;
        const int64_t l = find_list(a.tile_start, a.L, item);
        const int64_t m = item - a.tile_start[l];
        const int64_t ls = a.segoff[l * a.nch], le = a.segoff[(l + 1) * a.nch];
        ti.kind = 0;
        ti.j = l % a.nblk;
        ti.hk = (int)((l / a.nblk) % a.Hkv);
        ti.b = (int)(l / (a.nblk * a.Hkv));
        ti.e0 = ls + m * MOBA_TILE;
        ti.ne = (le - ti.e0 < MOBA_TILE) ? le - ti.e0 : MOBA_TILE;
        ti.klo = ti.j * a.bs;
        ti.khi = ti.klo + a.bs;
        ti.hq = 0;
        ti.t0 = 0;
        ti.nt = 0;
        return ti;
    }
    const int64_t d = item - a.Pmax;
    if (d >= a.D) return ti;
    const int64_t bh = d / a.per_bh, r = d % a.per_bh;
    ti.b = (int)(bh / a.Hq);
    ti.hq = (int)(bh % a.Hq);
    ti.hk = ti.hq / a.G;
    int64_t c = r / a.mb, m = r % a.mb;
    if (c >= a.nblk) {  // only reachable when the last block has fewer tiles
        c = a.nblk - 1;
        m = r - (a.nblk - 1) * a.mb;
    }
    const int64_t bstart = c * a.bs;
    const int64_t bend = (bstart + a.bs < a.N) ? bstart + a.bs : a.N;
    ti.kind = 1;
    ti.t0 = bstart + m * MOBA_TILE;
    ti.nt = (bend - ti.t0 < MOBA_TILE) ? bend - ti.t0 : MOBA_TILE;
    ti.klo = a.dense ? 0 : bstart;
    ti.khi = ti.t0 + ti.nt;
    ti.j = c;
    ti.e0 = 0;
    ti.ne = 0;
    return ti;
}
