// k_invert.cuh - inversion of the per-query selection into per-block query lists.
//
// The pages' FlashAttention pipeline ("MoBA tech-report summary", section 2,
// implementation steps 1-2) groups the queries by the key block they chose so
// that each block is attended once for all of its queries. Here that grouping
// is a stable-size counting sort keyed by list l = (b * Hkv + hk) * nblk + j:
//   count  : per (b, hk, token chunk) a shared-memory histogram over j,
//   scan   : exclusive prefix over counts[l][chunk] (list-major order),
//   scatter: each chunk writes its entries into its own segment of list l.
// An entry packs (t, query head, slot) where slot = position of j in the
// query's ascending selection row; only earlier blocks (j < c(t)) are listed,
// the own block is handled by the diagonal tiles.
//
// Integer work, HBM bound: the selection is read twice, entries written once.
#pragma once
#include "common.cuh"

#define INV_THREADS 256
#define INV_CHUNK 4096

__device__ __forceinline__ uint64_t pack_entry(int64_t t, int hq, int slot) {
    return (uint64_t)(uint32_t)t | ((uint64_t)(uint32_t)hq << 32) | ((uint64_t)(uint32_t)slot << 48);
}
__device__ __forceinline__ int64_t entry_t(uint64_t e) { return (int64_t)(uint32_t)e; }
__device__ __forceinline__ int entry_hq(uint64_t e) { return (int)((e >> 32) & 0xFFFF); }
__device__ __forceinline__ int entry_slot(uint64_t e) { return (int)(e >> 48); }

// Number of earlier blocks in a well-formed selection row (ascending distinct
// ids < c, then c, then only -1), or -1 if the row is malformed.
__device__ __forceinline__ int check_row(const int32_t* row, int topk, int64_t c) {
    int p = -1;
    int64_t prev = -1;
    for (int i = 0; i < topk; ++i) {
        int32_t j = row[i];
        if (p < 0) {
            if (j == c) {
                p = i;
            } else if (j < 0 || j > c || j <= prev) {
                return -1;
            }
            prev = j;
        } else if (j != -1) {
            return -1;
        }
    }
    return p;
}

// grid (nch, Hkv, B); dynamic smem: nblk u32 counters.
__global__ void __launch_bounds__(INV_THREADS) moba_count_kernel(const int32_t* __restrict__ idx,
                                                                 uint32_t* __restrict__ counts, int64_t N,
                                                                 int Hq, int Hkv, int bs, int topk,
                                                                 int64_t nblk, int64_t nch) {
    extern __shared__ uint32_t hist[];
    const int64_t ch = blockIdx.x;
    const int hk = blockIdx.y, b = blockIdx.z;
    const int G = Hq / Hkv;
    for (int64_t j = threadIdx.x; j < nblk; j += INV_THREADS) hist[j] = 0;
    __syncthreads();
    const int64_t t0 = ch * INV_CHUNK;
    const int64_t tn = (t0 + INV_CHUNK < N ? t0 + INV_CHUNK : N) - t0;
    for (int64_t r = threadIdx.x; r < tn * G; r += INV_THREADS) {
        const int g = (int)(r / tn);
        const int64_t t = t0 + r % tn;
        const int hq = hk * G + g;
        const int32_t* row = idx + (((int64_t)b * Hq + hq) * N + t) * topk;
        const int64_t c = t / bs;
        const int p = check_row(row, topk, c);
        for (int i = 0; i < p; ++i) atomicAdd(&hist[row[i]], 1u);
    }
    __syncthreads();
    const int64_t lbase = ((int64_t)b * Hkv + hk) * nblk;
    for (int64_t j = threadIdx.x; j < nblk; j += INV_THREADS) counts[(lbase + j) * nch + ch] = hist[j];
}

// grid (nch, Hkv, B); dynamic smem: nblk u32 cursors + nblk i64 bases.
__global__ void __launch_bounds__(INV_THREADS) moba_scatter_kernel(const int32_t* __restrict__ idx,
                                                                   const int64_t* __restrict__ segoff,
                                                                   uint64_t* __restrict__ entries, int64_t N,
                                                                   int Hq, int Hkv, int bs, int topk,
                                                                   int64_t nblk, int64_t nch) {
    extern __shared__ int64_t sbase[];
    uint32_t* cur = reinterpret_cast<uint32_t*>(sbase + nblk);
    const int64_t ch = blockIdx.x;
    const int hk = blockIdx.y, b = blockIdx.z;
    const int G = Hq / Hkv;
    const int64_t lbase = ((int64_t)b * Hkv + hk) * nblk;
    for (int64_t j = threadIdx.x; j < nblk; j += INV_THREADS) {
        sbase[j] = segoff[(lbase + j) * nch + ch];
        cur[j] = 0;
    }
    __syncthreads();
    const int64_t t0 = ch * INV_CHUNK;
    const int64_t tn = (t0 + INV_CHUNK < N ? t0 + INV_CHUNK : N) - t0;
    for (int64_t r = threadIdx.x; r < tn * G; r += INV_THREADS) {
        const int g = (int)(r / tn);
        const int64_t t = t0 + r % tn;
        const int hq = hk * G + g;
        const int32_t* row = idx + (((int64_t)b * Hq + hq) * N + t) * topk;
        const int64_t c = t / bs;
        const int p = check_row(row, topk, c);
        for (int i = 0; i < p; ++i) {
            const int32_t j = row[i];
            const uint32_t k = atomicAdd(&cur[j], 1u);
            entries[sbase[j] + k] = pack_entry(t, hq, i);
        }
    }
}

// ---------------------------------------------------------------- exclusive scan (u32 -> i64)
#define SCAN_THREADS 256
#define SCAN_PER_THREAD 8
#define SCAN_TILE (SCAN_THREADS * SCAN_PER_THREAD)

// Value i of the scan input: either counts[i] or, for the work items, the
// number of 256-row tile pairs of list i computed from the list offsets.
struct ScanSrc {
    const uint32_t* vals;    // direct values, or null
    const int64_t* segoff;   // list offsets (stride nch) when vals is null
    int64_t nch;
    __device__ __forceinline__ int64_t get(int64_t i) const {
        if (vals) return vals[i];
        int64_t len = segoff[(i + 1) * nch] - segoff[i * nch];
        return (len + 2 * MOBA_TILE - 1) / (2 * MOBA_TILE);
    }
};

__device__ __forceinline__ int64_t block_excl_scan(int64_t v, int64_t* total) {
    __shared__ int64_t warp_sums[SCAN_THREADS / 32];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    int64_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int64_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[w] = x;
    __syncthreads();
    if (w == 0) {
        int64_t s = (lane < SCAN_THREADS / 32) ? warp_sums[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int64_t y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        if (lane < SCAN_THREADS / 32) warp_sums[lane] = s;
    }
    __syncthreads();
    int64_t before = (w > 0 ? warp_sums[w - 1] : 0) + x - v;
    *total = warp_sums[SCAN_THREADS / 32 - 1];
    __syncthreads();
    return before;
}

__global__ void __launch_bounds__(SCAN_THREADS) moba_scan_partial_kernel(ScanSrc src, int64_t n,
                                                                         int64_t* __restrict__ part) {
    const int64_t base = (int64_t)blockIdx.x * SCAN_TILE + (int64_t)threadIdx.x * SCAN_PER_THREAD;
    int64_t s = 0;
#pragma unroll
    for (int i = 0; i < SCAN_PER_THREAD; ++i)
        if (base + i < n) s += src.get(base + i);
    int64_t tot;
    block_excl_scan(s, &tot);
    if (threadIdx.x == 0) part[blockIdx.x] = tot;
}

// One CTA: exclusive scan of the per-tile sums in place.
__global__ void __launch_bounds__(SCAN_THREADS) moba_scan_top_kernel(int64_t* __restrict__ part, int64_t nparts) {
    int64_t carry = 0;
    for (int64_t b0 = 0; b0 < nparts; b0 += SCAN_THREADS) {
        int64_t i = b0 + threadIdx.x;
        int64_t v = (i < nparts) ? part[i] : 0;
        int64_t tot;
        int64_t ex = block_excl_scan(v, &tot);
        if (i < nparts) part[i] = carry + ex;
        carry += tot;
    }
}

__global__ void __launch_bounds__(SCAN_THREADS) moba_scan_final_kernel(ScanSrc src, int64_t n,
                                                                       const int64_t* __restrict__ part,
                                                                       int64_t* __restrict__ out) {
    const int64_t base = (int64_t)blockIdx.x * SCAN_TILE + (int64_t)threadIdx.x * SCAN_PER_THREAD;
    int64_t v[SCAN_PER_THREAD];
    int64_t s = 0;
#pragma unroll
    for (int i = 0; i < SCAN_PER_THREAD; ++i) {
        v[i] = (base + i < n) ? src.get(base + i) : 0;
        s += v[i];
    }
    int64_t tot;
    int64_t ex = block_excl_scan(s, &tot) + part[blockIdx.x];
#pragma unroll
    for (int i = 0; i < SCAN_PER_THREAD; ++i) {
        if (base + i < n) out[base + i] = ex;
        ex += v[i];
    }
    if (blockIdx.x == gridDim.x - 1 && threadIdx.x == SCAN_THREADS - 1) out[n] = part[blockIdx.x] + tot;
}
