// k_decode.cuh - one decode step of MoBA: the newest query of each sequence
// (position L - 1) against its KV cache, with the same gate as the prefill.
//
// The step is the prefill's definition at the last row ("MoBA project hub",
// Steps 2-3; "MoBA tech-report summary", section 2): the query scores every
// earlier full block j < c = floor((L-1) / bs) as <q, Kbar_j>, keeps its own
// block c and the topk - 1 best earlier ones (lower index on equal scores),
// and attends their keys (the own block up to L - 1). A full-attention layer
// of a hybrid model ("KIMI MoBA" blog, section 3, hybrid_layers; the pages run
// decode with full attention) keeps every block.
//
// Three kernels:
//   select  one CTA per (b, kv head): exact fp64 scores of the G query heads
//           against the cached block summaries Kbar, top-k per head, then the
//           union of the group's kept blocks with a G-bit mask per block (the
//           heads that kept it), so each K/V block is read once for the group;
//   attend  one CTA per (b, kv head, union entry, 512-key chunk): streams the
//           chunk's keys and values through shared memory once and keeps an
//           online softmax (max, sum, 128 outputs) for every head that kept the
//           block; writes one partial per head;
//   merge   one CTA per (b, query head): log-sum-exp merge of its partials.
// Memory bound: the K/V bytes of the union blocks dominate.
#pragma once
#include "common.cuh"

#define DEC_THREADS 128
#define DEC_CHUNK 512       // keys per attend CTA
#define DEC_TILE 64         // keys per shared-memory tile
#define DEC_MAX_G 16        // query heads per kv head (static shared memory of the attend kernel)
#define DEC_PART (MOBA_D + 2)  // one partial: m (log2 units), l, o[128]
#define DEC_KSTRIDE (MOBA_D + 2)  // K tile row stride in bf16: 65 words, so lanes reading one feature
                                  // of 32 different keys hit 32 different banks

struct DecodeParams {
    const uint16_t* q;    // [B, Hq, d]
    const uint16_t* k;    // [B, Lmax, Hkv, d]
    const uint16_t* v;
    const double* kbar;   // [B, Hkv, kbar_rows, d], block summaries of full blocks 0 .. floor(L/bs) - 1
    int64_t kbar_rows;    // rows per (b, kv head) in kbar
    int64_t L, Lmax;
    int B, Hq, Hkv, G, bs, topk;
    int64_t c;            // own block of the query
    int64_t umax;         // union capacity per (b, kv head)
    int64_t nch;          // chunks per block
    int full;             // keep every block
    int32_t* ucount;      // [B*Hkv]
    int32_t* ulist;       // [B*Hkv][umax] block ids, ascending
    uint32_t* umask;      // [B*Hkv][umax] heads of the group that kept the block
    float* part;          // [B*Hkv][umax][nch][G][DEC_PART]
    int32_t* idx_out;     // optional [B, Hq, topk]
    uint16_t* out;        // [B, Hq, d]
    float* lse;           // [B, Hq]
    float scale_log2;     // log2(e) / sqrt(d)
};

// ---------------------------------------------------------------- select
// dynamic smem: c doubles (scores of one head) + G * topk ints (kept blocks per head)
__global__ void __launch_bounds__(DEC_THREADS) moba_decode_select_kernel(const DecodeParams p) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int hk = blockIdx.x, b = blockIdx.y;
    const int64_t c = p.c;
    const int kp = p.topk - 1;
    const int64_t bh0 = (int64_t)blockIdx.y * p.Hkv + blockIdx.x;
    if (p.full) {  // every block 0 .. c is kept by every head
        const uint32_t all = (1u << p.G) - 1u;
        for (int64_t j = threadIdx.x; j <= c; j += DEC_THREADS) {
            p.ulist[bh0 * p.umax + j] = (int32_t)j;
            p.umask[bh0 * p.umax + j] = all;
        }
        if (threadIdx.x == 0) p.ucount[bh0] = (int32_t)(c + 1);
        return;
    }
    const int64_t npast = c < kp ? c : kp;  // earlier blocks kept per head
    double* sc = (double*)smem;
    int32_t* kept = (int32_t*)(smem + sizeof(double) * (c > 0 ? c : 1));  // [G][npast]
    __shared__ double rs[DEC_THREADS / 32];
    __shared__ int32_t rj[DEC_THREADS / 32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t bh = (int64_t)b * p.Hkv + hk;

    for (int g = 0; g < p.G; ++g) {
        const int hq = hk * p.G + g;
        int32_t* kg = kept + (int64_t)g * (npast > 0 ? npast : 1);
        if (c <= kp) {  // every earlier block is kept
            for (int64_t j = threadIdx.x; j < npast; j += DEC_THREADS) kg[j] = (int32_t)j;
            continue;
        }
        // exact fp64 scores <q, Kbar_j>, features ascending (one fused multiply-add each)
        const uint16_t* qr = p.q + ((int64_t)b * p.Hq + hq) * MOBA_D;
        for (int64_t j = threadIdx.x; j < c; j += DEC_THREADS) {
            const double* kb = p.kbar + (bh * p.kbar_rows + j) * MOBA_D;
            double s = 0.0;
#pragma unroll 8
            for (int e = 0; e < MOBA_D; ++e) s = fma((double)bf16_bits_to_float(qr[e]), kb[e], s);
            sc[j] = s;
        }
        __syncthreads();
        // kp rounds of a block-wide arg-max over (score desc, index asc); the winner is struck out
        for (int r = 0; r < kp; ++r) {
            double best = -INFINITY;
            int32_t bj = 0x7FFFFFFF;
            for (int64_t j = threadIdx.x; j < c; j += DEC_THREADS) {
                const double s = sc[j];
                if (s > best || (s == best && (int32_t)j < bj)) {
                    best = s;
                    bj = (int32_t)j;
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const double s2 = __shfl_xor_sync(0xffffffffu, best, o);
                const int32_t j2 = __shfl_xor_sync(0xffffffffu, bj, o);
                if (s2 > best || (s2 == best && j2 < bj)) {
                    best = s2;
                    bj = j2;
                }
            }
            if (lane == 0) {
                rs[warp] = best;
                rj[warp] = bj;
            }
            __syncthreads();
            if (threadIdx.x == 0) {
                for (int w = 1; w < DEC_THREADS / 32; ++w)
                    if (rs[w] > best || (rs[w] == best && rj[w] < bj)) {
                        best = rs[w];
                        bj = rj[w];
                    }
                kg[r] = bj;
                sc[bj] = -INFINITY;  // struck out (real scores are finite)
            }
            __syncthreads();
        }
    }
    __syncthreads();
    if (threadIdx.x != 0) return;
    // per head: ascending kept blocks (own block last) into idx_out, then the union of the group
    for (int g = 0; g < p.G; ++g) {
        int32_t* kg = kept + (int64_t)g * (npast > 0 ? npast : 1);
        for (int64_t i = 1; i < npast; ++i) {  // insertion sort (npast <= topk - 1)
            const int32_t x = kg[i];
            int64_t u = i;
            while (u > 0 && kg[u - 1] > x) {
                kg[u] = kg[u - 1];
                --u;
            }
            kg[u] = x;
        }
        if (p.idx_out) {
            int32_t* orow = p.idx_out + ((int64_t)b * p.Hq + hk * p.G + g) * p.topk;
            for (int i = 0; i < p.topk; ++i) orow[i] = i < npast ? kg[i] : (i == npast ? (int32_t)c : -1);
        }
    }
    // union: a G-way merge of the sorted lists, then the own block
    int32_t* ul = p.ulist + bh * p.umax;
    uint32_t* um = p.umask + bh * p.umax;
    int64_t n = 0;
    int64_t pos[DEC_MAX_G];
    for (int g = 0; g < p.G; ++g) pos[g] = 0;
    for (;;) {
        int32_t j = 0x7FFFFFFF;
        for (int g = 0; g < p.G; ++g)
            if (pos[g] < npast) {
                const int32_t x = kept[(int64_t)g * npast + pos[g]];
                if (x < j) j = x;
            }
        if (j == 0x7FFFFFFF) break;
        uint32_t mask = 0;
        for (int g = 0; g < p.G; ++g)
            if (pos[g] < npast && kept[(int64_t)g * npast + pos[g]] == j) {
                mask |= 1u << g;
                ++pos[g];
            }
        ul[n] = j;
        um[n] = mask;
        ++n;
    }
    ul[n] = (int32_t)c;  // the own block, kept by every head
    um[n] = (1u << p.G) - 1u;
    ++n;
    p.ucount[bh] = (int32_t)n;
}

// ---------------------------------------------------------------- attend
// grid (umax * nch, Hkv, B); static smem: K and V tiles, the heads' queries, scores and state.
// GM >= G (query heads per kv head) is a template argument so each thread's outputs stay in
// registers; heads g >= G are never in a block's mask and are skipped.
template <int GM>
__global__ void __launch_bounds__(DEC_THREADS) moba_decode_attend_kernel(const DecodeParams p) {
    const int hk = blockIdx.y, b = blockIdx.z;
    const int64_t bh = (int64_t)b * p.Hkv + hk;
    const int64_t u = blockIdx.x / p.nch, ch = blockIdx.x % p.nch;
    if (u >= p.ucount[bh]) return;
    const int64_t j = p.ulist[bh * p.umax + u];
    const uint32_t mask = p.umask[bh * p.umax + u];
    const int64_t bend = (j == p.c) ? p.L : (j + 1) * p.bs;  // keys [j*bs, bend)
    const int64_t k0 = j * p.bs + ch * DEC_CHUNK;
    const int64_t k1 = (k0 + DEC_CHUNK < bend) ? k0 + DEC_CHUNK : bend;

    __shared__ __align__(16) uint16_t sk[DEC_TILE][DEC_KSTRIDE];
    __shared__ __align__(16) uint16_t sv[DEC_TILE][MOBA_D];
    __shared__ float sq[GM][MOBA_D];
    __shared__ float sp[GM][DEC_TILE];
    __shared__ float sm[GM], sl[GM], sa[GM];
    const int G = p.G;
    for (int i = threadIdx.x; i < G * MOBA_D; i += DEC_THREADS) {
        const int g = i / MOBA_D, e = i % MOBA_D;
        sq[g][e] = bf16_bits_to_float(p.q[((int64_t)b * p.Hq + hk * G + g) * MOBA_D + e]);
    }
    if (threadIdx.x < G) {
        sm[threadIdx.x] = -INFINITY;
        sl[threadIdx.x] = 0.f;
    }
    float o[GM];  // this thread's output feature e = threadIdx.x, per head
#pragma unroll
    for (int g = 0; g < GM; ++g) o[g] = 0.f;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int64_t t0 = k0; t0 < k1; t0 += DEC_TILE) {
        const int nk = (int)((k1 - t0 < DEC_TILE) ? k1 - t0 : DEC_TILE);
        __syncthreads();  // the previous tile is no longer read
        for (int i = threadIdx.x; i < DEC_TILE * (MOBA_D / 8); i += DEC_THREADS) {
            const int kk = i / (MOBA_D / 8), c8 = i % (MOBA_D / 8);
            uint4 kw = make_uint4(0u, 0u, 0u, 0u), vw = kw;
            if (kk < nk) {
                const int64_t row = ((int64_t)b * p.Lmax + t0 + kk) * p.Hkv + hk;
                kw = ld_nc_v4(p.k + row * MOBA_D + c8 * 8);
                vw = ld_nc_v4(p.v + row * MOBA_D + c8 * 8);
            }
            uint32_t* kd = reinterpret_cast<uint32_t*>(&sk[kk][c8 * 8]);  // 4-byte aligned rows
            kd[0] = kw.x;
            kd[1] = kw.y;
            kd[2] = kw.z;
            kd[3] = kw.w;
            *reinterpret_cast<uint4*>(&sv[kk][c8 * 8]) = vw;
        }
        __syncthreads();
        // scores: thread (kk = t % 64) for heads g = t / 64, t / 64 + 2, ...
        {
            const int kk = threadIdx.x % DEC_TILE;
            for (int g = threadIdx.x / DEC_TILE; g < G; g += DEC_THREADS / DEC_TILE) {
                float s = -INFINITY;
                if (kk < nk && ((mask >> g) & 1u)) {
                    float acc = 0.f;
#pragma unroll 16
                    for (int e = 0; e < MOBA_D; e += 2) {
                        const uint32_t w = *reinterpret_cast<const uint32_t*>(&sk[kk][e]);
                        acc = fmaf(sq[g][e], bf16lo(w), acc);
                        acc = fmaf(sq[g][e + 1], bf16hi(w), acc);
                    }
                    s = acc * p.scale_log2;
                }
                sp[g][kk] = s;
            }
        }
        __syncthreads();
        // online softmax per head: warp w handles heads w, w + 4, ...
        for (int g = warp; g < G; g += DEC_THREADS / 32) {
            if (!((mask >> g) & 1u)) continue;
            const float s0 = sp[g][lane], s1 = sp[g][lane + 32];
            float mx = fmaxf(s0, s1);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            const float m_old = sm[g];
            const float m_new = fmaxf(m_old, mx);  // finite: every tile holds at least one key
            const float p0 = exp2f(s0 - m_new), p1 = exp2f(s1 - m_new);
            float sum = p0 + p1;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
            sp[g][lane] = p0;
            sp[g][lane + 32] = p1;
            __syncwarp();
            if (lane == 0) {
                const float a = exp2f(m_old - m_new);  // 0 on the first tile (m_old = -inf)
                sa[g] = a;
                sl[g] = sl[g] * a + sum;
                sm[g] = m_new;
            }
        }
        __syncthreads();
        // outputs: thread e accumulates feature e of every head that kept the block
        const int e = threadIdx.x;
#pragma unroll
        for (int g = 0; g < GM; ++g) {
            if (!((mask >> g) & 1u)) continue;  // also every g >= G
            float acc = o[g] * sa[g];
            for (int kk = 0; kk < nk; ++kk) acc = fmaf(sp[g][kk], bf16_bits_to_float(sv[kk][e]), acc);
            o[g] = acc;
        }
    }
    __syncthreads();
    // partial per head that kept the block (an empty chunk writes l = 0)
#pragma unroll
    for (int g = 0; g < GM; ++g) {
        if (!((mask >> g) & 1u)) continue;  // also every g >= G
        float* pr = p.part + (((bh * p.umax + u) * p.nch + ch) * G + g) * DEC_PART;
        const bool empty = k1 <= k0;
        if (threadIdx.x == 0) {
            pr[0] = empty ? -INFINITY : sm[g];
            pr[1] = empty ? 0.f : sl[g];
        }
        pr[2 + threadIdx.x] = empty ? 0.f : o[g];
    }
}

// ---------------------------------------------------------------- merge
// grid (Hq, B): out = sum_i 2^(m_i - M) o_i / sum_i 2^(m_i - M) l_i over the head's partials.
__global__ void __launch_bounds__(DEC_THREADS) moba_decode_merge_kernel(const DecodeParams p) {
    const int hq = blockIdx.x, b = blockIdx.y;
    const int hk = hq / p.G, g = hq % p.G;
    const int64_t bh = (int64_t)b * p.Hkv + hk;
    const int n = p.ucount[bh];
    float M = -INFINITY;
    for (int u = 0; u < n; ++u) {
        if (!((p.umask[bh * p.umax + u] >> g) & 1u)) continue;
        for (int64_t ch = 0; ch < p.nch; ++ch) {
            const float* pr = p.part + (((bh * p.umax + u) * p.nch + ch) * p.G + g) * DEC_PART;
            if (pr[1] > 0.f) M = fmaxf(M, pr[0]);
        }
    }
    float acc = 0.f, lsum = 0.f;
    const int e = threadIdx.x;
    for (int u = 0; u < n; ++u) {
        if (!((p.umask[bh * p.umax + u] >> g) & 1u)) continue;
        for (int64_t ch = 0; ch < p.nch; ++ch) {
            const float* pr = p.part + (((bh * p.umax + u) * p.nch + ch) * p.G + g) * DEC_PART;
            if (!(pr[1] > 0.f)) continue;
            const float w = exp2f(pr[0] - M);
            lsum = fmaf(w, pr[1], lsum);
            acc = fmaf(w, pr[2 + e], acc);
        }
    }
    const float inv = 1.f / lsum;
    p.out[((int64_t)b * p.Hq + hq) * MOBA_D + e] = __bfloat16_as_ushort(__float2bfloat16_rn(acc * inv));
    if (e == 0) p.lse[(int64_t)b * p.Hq + hq] = (M + __log2f(lsum)) * 0.69314718055994530942f;
}
