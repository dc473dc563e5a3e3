// k_attn_common.cuh - work decomposition shared by the attention kernels.
//
// A work item is a PAIR of 128-row query tiles that read the same keys, so
// one stream of K/V steps feeds both (the tensor-core kernel alternates
// between them while the other's softmax runs):
//   [0, P)           past-block pairs: up to 256 consecutive entries of one
//                    query list l = (b, hk, j); both tiles attend all keys of
//                    block j without a mask; results are partials (O normalised
//                    by its own sum, lse) stored in each entry's slot.
//   [Pmax, Pmax + D) own-block ("diagonal") pairs: tiles 2m and 2m + 1 of the
//                    128-token tiles of one query head inside one block c; key
//                    range c*bs .. last token of the tile, causal mask; the
//                    partial goes to out / lse and is merged later. In dense
//                    mode the key range starts at 0 and the result is final.
// The second tile of a pair may be missing (odd tile count); P (the real
// number of past pairs) is only known on the device and items in [P, Pmax)
// are empty.
#pragma once
#include "common.cuh"
#include "k_invert.cuh"

#define MOBA_PAIR_ROWS (2 * MOBA_TILE)

// A past pair as one 16-byte record, so that a role decodes an item with one load that does
// not depend on another (and can be issued an item ahead): its first entry, its list
// l = (b, hk, j) and its entry count (1..256). e0 < 0 marks an empty item (P <= p < Pmax).
struct __align__(16) PairDesc {
    int64_t e0;
    int32_t l;
    int32_t n;
};

struct AttnParams {
    const uint16_t* q;
    const uint16_t* k;
    const uint16_t* v;
    int64_t N;
    int B, Hq, Hkv, G, bs, topk, kp;
    int64_t nblk, nch;
    // past pairs
    const uint64_t* entries;
    const int64_t* segoff;      // list l spans entries [segoff[l*nch], segoff[(l+1)*nch])
    const PairDesc* pairs;       // descriptor of each past pair, [Pmax]
    int64_t L, Pmax;
    uint16_t* opart;  // bf16 [B, Hq, N, kp, d]
    float* lpart;     // fp32 [B, Hq, N, kp]
    // diagonal / dense pairs
    int64_t D;
    int64_t mb, ml, per_bh;  // tiles per full block, in the last block, pairs per (b, hq)
    int dense;               // 1: dense causal attention, key range starts at 0
    uint16_t* out;           // bf16 [B, N, Hq, d]
    float* lse;              // fp32 [B, Hq, N]
    float scale_log2;        // log2(e) / sqrt(d)
};

// Largest l with tile_start[l] <= p (lists without pairs are skipped).
__device__ __forceinline__ int64_t find_list(const int64_t* __restrict__ ts, int64_t L, int64_t p) {
    int64_t lo = 0, hi = L;  // invariant: ts[lo] <= p < ts[hi]
    while (hi - lo > 1) {
        int64_t mid = (lo + hi) >> 1;
        if (ts[mid] <= p) lo = mid;
        else hi = mid;
    }
    return lo;
}

// pairs[p] for every p < Pmax from the per-list pair prefix ts (ts[L] = P) and the list
// bounds segoff (list l spans entries [segoff[l*nch], segoff[(l+1)*nch])).
__global__ void __launch_bounds__(256) moba_item_list_kernel(const int64_t* __restrict__ ts,
                                                             const int64_t* __restrict__ segoff, int64_t L,
                                                             int64_t nch, int64_t Pmax, PairDesc* __restrict__ pairs) {
    const int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (p >= Pmax) return;
    PairDesc d;
    d.e0 = -1;
    d.l = 0;
    d.n = 0;
    if (p < ts[L]) {
        const int64_t l = find_list(ts, L, p);
        const int64_t le = segoff[(l + 1) * nch];
        d.e0 = segoff[l * nch] + (p - ts[l]) * MOBA_PAIR_ROWS;
        d.l = (int32_t)l;
        d.n = (int32_t)((le - d.e0 < MOBA_PAIR_ROWS) ? le - d.e0 : MOBA_PAIR_ROWS);
    }
    pairs[p] = d;
}

struct TileInfo {
    int kind;         // 0 = past, 1 = diagonal / dense, -1 = no tile
    int b, hk;
    int64_t j;        // key block of a past tile
    int64_t e0, ne;   // past: first entry and count
    int hq;           // diagonal: query head
    int64_t t0, nt;   // diagonal: first token and count
    int64_t klo;      // first key
    int64_t khi;      // one past the last key any row of the tile reads
};

__device__ __forceinline__ int64_t tile_steps(const TileInfo& ti) {
    return ti.kind < 0 ? 0 : (ti.khi - ti.klo + MOBA_KCHUNK - 1) / MOBA_KCHUNK;
}

struct PairInfo {
    TileInfo t[2];
    int64_t ns;  // K/V steps of the pair = the longer tile's steps
};

// The descriptor of an item (a dummy for own-block items, whose decoding is arithmetic only).
__device__ __forceinline__ PairDesc pair_desc(const AttnParams& a, int64_t item) {
    if (item < a.Pmax) return a.pairs[item];
    PairDesc d;
    d.e0 = -1;
    d.l = 0;
    d.n = 0;
    return d;
}

__device__ __forceinline__ PairInfo decode_pair(const AttnParams& a, int64_t item, const PairDesc pd) {
    PairInfo pi;
    pi.t[0].kind = -1;
    pi.t[1].kind = -1;
    pi.ns = 0;
    if (item < a.Pmax) {
        if (pd.e0 < 0) return pi;
        const int64_t l = pd.l;
        const int64_t j = l % a.nblk;
        const int hk = (int)((l / a.nblk) % a.Hkv);
        const int b = (int)(l / (a.nblk * a.Hkv));
#pragma unroll
        for (int x = 0; x < 2; ++x) {
            TileInfo& ti = pi.t[x];
            if (x * MOBA_TILE >= pd.n) continue;
            ti.kind = 0;
            ti.j = j;
            ti.hk = hk;
            ti.b = b;
            ti.e0 = pd.e0 + x * MOBA_TILE;
            ti.ne = (pd.n - x * MOBA_TILE < MOBA_TILE) ? pd.n - x * MOBA_TILE : MOBA_TILE;
            ti.klo = j * a.bs;
            ti.khi = ti.klo + a.bs;
            ti.hq = 0;
            ti.t0 = 0;
            ti.nt = 0;
        }
    } else {
        const int64_t d = item - a.Pmax;
        if (d >= a.D) return pi;
        const int64_t bh = d / a.per_bh, r = d % a.per_bh;
        const int64_t pb = (a.mb + 1) / 2;  // pairs per full block
        int64_t c = r / pb, m = r % pb;
        if (c >= a.nblk - 1) {  // the last block may have fewer tiles
            c = a.nblk - 1;
            m = r - (a.nblk - 1) * pb;
        }
        const int64_t bstart = c * a.bs;
        const int64_t bend = (bstart + a.bs < a.N) ? bstart + a.bs : a.N;
#pragma unroll
        for (int x = 0; x < 2; ++x) {
            TileInfo& ti = pi.t[x];
            const int64_t t0 = bstart + (2 * m + x) * MOBA_TILE;
            if (t0 >= bend) continue;
            ti.kind = 1;
            ti.b = (int)(bh / a.Hq);
            ti.hq = (int)(bh % a.Hq);
            ti.hk = ti.hq / a.G;
            ti.t0 = t0;
            ti.nt = (bend - t0 < MOBA_TILE) ? bend - t0 : MOBA_TILE;
            ti.klo = a.dense ? 0 : bstart;
            ti.khi = t0 + ti.nt;
            ti.j = c;
            ti.e0 = 0;
            ti.ne = 0;
        }
    }
    const int64_t n0 = tile_steps(pi.t[0]), n1 = tile_steps(pi.t[1]);
    pi.ns = n0 > n1 ? n0 : n1;
    return pi;
}

__device__ __forceinline__ PairInfo decode_pair(const AttnParams& a, int64_t item) {
    return decode_pair(a, item, pair_desc(a, item));
}
