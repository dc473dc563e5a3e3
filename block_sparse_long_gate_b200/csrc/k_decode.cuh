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
// Four kernels:
//   select  one CTA per query head: exact fp64 scores against the cached block
//           summaries Kbar into shared memory (a warp per summary row, coalesced);
//           each warp keeps the best topk - 1 of a slice of the blocks by counting,
//           for each block, the blocks of the slice that rank before it; the head's
//           topk - 1 are the warps' winners of rank < topk - 1 among all of them;
//   union   one CTA per (b, kv head): the union of the group's kept blocks in
//           ascending order with a G-bit mask per block (the heads that kept it),
//           so each K/V block is read once for the whole group;
//   attend  one CTA per (b, kv head, union entry, chunk of 512 to 4096 keys), four
//           warps of a quarter chunk each. A warp streams its keys and values through its own
//           3-stage cp.async ring of 16-key stages and runs both products on the
//           tensor cores (mma.sync m16n8k16, bf16 in, fp32 accumulate) with the
//           group's heads as the 16 rows: S = Q K^T, an online softmax per row,
//           O += P V. The four warps' states are combined in shared memory into
//           one partial per head that kept the block;
//   merge   one CTA per (b, query head): log-sum-exp merge of its partials, the
//           warps splitting the partials.
// Memory bound: the K/V bytes of the union blocks dominate.
//
// union, attend and merge are launched as programmatic dependents of the kernel before them
// (the launch overlaps that kernel's tail): each waits for its predecessor's results with
// griddepcontrol.wait before reading them, and attend loads its queries (the caller's input,
// complete before select started) before it waits. Launched plainly, both instructions do nothing.
#pragma once
#include "common.cuh"

__device__ __forceinline__ void dec_wait_prior_grid() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void dec_allow_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

#define DEC_MAX_G 16        // query heads per kv head: the 16 rows of an m16n8k16 product
#define DEC_SEL_THREADS 512
#define DEC_SEL_WARPS (DEC_SEL_THREADS / 32)
#define DEC_UNION_THREADS 256
#define DEC_WARPS 4
#define DEC_MIN_CHUNK 512                           // keys per attend CTA, at least (the host may double it)
#define DEC_SKEYS 16                                // keys per ring stage
#define DEC_STAGES 3
#define DEC_ROW 272  // bytes per staged key row: 256 + 16, so the 8 rows one ldmatrix reads hit distinct banks
#define DEC_STAGE_BYTES (2 * DEC_SKEYS * DEC_ROW)   // K rows, then V rows
#define DEC_ATTEND_SMEM (DEC_WARPS * DEC_STAGES * DEC_STAGE_BYTES)
#define DEC_MERGE_THREADS 256
#define DEC_PART 132  // one partial: m (log2 units), l, 2 unused, o[128] (16-byte aligned)

static_assert(DEC_WARPS * 32 == MOBA_D, "the combine gives each thread one output feature");
static_assert(DEC_WARPS * DEC_MAX_G * (MOBA_D + 2) * 4 <= DEC_ATTEND_SMEM, "combine area exceeds the rings");

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
    int64_t chunk;        // keys per attend CTA (a multiple of DEC_WARPS * DEC_SKEYS)
    int64_t nch;          // chunks per block
    int full;             // keep every block
    int32_t* kept;        // [B*Hkv][G][max(topk - 1, 1)] kept earlier blocks per head, ascending
    int32_t* ucount;      // [B*Hkv]
    int32_t* ulist;       // [B*Hkv][umax] block ids, ascending
    uint32_t* umask;      // [B*Hkv][umax] heads of the group that kept the block
    float* part;          // [B*Hkv][umax][nch][G][DEC_PART]
    int32_t* idx_out;     // optional [B, Hq, topk]
    uint16_t* out;        // [B, Hq, d]
    float* lse;           // [B, Hq]
    float scale_log2;     // log2(e) / sqrt(d)
};

// (score desc, block asc): does (s2, j2) rank before (s, j)?
__device__ __forceinline__ bool dec_before(double s2, int32_t j2, double s, int32_t j) {
    return s2 > s || (s2 == s && j2 < j);
}

// Rank of entry i among the n entries (sc[k], jd[k]) by dec_before: how many rank before it.
// The ranks of distinct blocks are distinct, so the entries of rank < m are the m best.
// Lanes of a warp that scan the same array read each entry at the same time (a broadcast).
__device__ __forceinline__ int dec_rank(const double* sc, const int32_t* jd, int n, double s, int32_t j) {
    int rank = 0;
    for (int k = 0; k < n; ++k) rank += dec_before(sc[k], jd[k], s, j);
    return rank;
}

// ---------------------------------------------------------------- select
// grid (G, Hkv, B); dynamic smem (when c > topk - 1 > 0): the c scores, two areas of
// DEC_SEL_WARPS (topk - 1) (score, block) candidates (the warps' lists and their compacted
// merge), then the c block ids.
__global__ void __launch_bounds__(DEC_SEL_THREADS) moba_decode_select_kernel(const DecodeParams p) {
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ int32_t cnt[DEC_SEL_WARPS];
    __shared__ int32_t fj[MOBA_MAX_TOPK];
    const int g = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
    const int hq = hk * p.G + g;
    const int64_t bh = (int64_t)b * p.Hkv + hk;
    const int64_t c = p.c;
    const int kp = p.topk - 1;
    const int npast = (int)(c < kp ? c : kp);  // earlier blocks kept
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int32_t* kept = p.kept + (bh * p.G + g) * (kp > 0 ? kp : 1);
    dec_allow_dependents();
    if (c > kp && kp > 0) {
        constexpr int NW = DEC_SEL_WARPS;
        double* sc = (double*)smem;                  // [c] scores
        double* cs = sc + c;                         // [NW][kp] candidate scores per warp
        double* ms = cs + NW * kp;                   // [NW kp] the compacted candidates
        int32_t* cj = (int32_t*)(ms + NW * kp);      // [NW][kp] candidate blocks per warp
        int32_t* mj = cj + NW * kp;                  // [NW kp]
        int32_t* sj = mj + NW * kp;                  // [c] block ids
        // exact fp64 scores <q, Kbar_j>: a warp per row, lane l multiplies features 4l .. 4l + 3
        // (fused multiply-adds in feature order), then a butterfly sum over the lanes. Eight rows
        // per warp are in flight at once. A NaN score ranks as -inf.
        constexpr int RW = 8;
        const uint16_t* qr = p.q + ((int64_t)b * p.Hq + hq) * MOBA_D + 4 * lane;
        const uint2 qw = *reinterpret_cast<const uint2*>(qr);
        const double q0 = bf16lo(qw.x), q1 = bf16hi(qw.x), q2 = bf16lo(qw.y), q3 = bf16hi(qw.y);
        const double* kb0 = p.kbar + bh * p.kbar_rows * MOBA_D + 4 * lane;
        for (int64_t j0 = warp; j0 < c; j0 += RW * NW) {
            double2 a[RW], bq[RW];
#pragma unroll
            for (int r = 0; r < RW; ++r) {
                const int64_t j = j0 + (int64_t)r * NW;
                a[r] = make_double2(0.0, 0.0);
                bq[r] = a[r];
                if (j < c) {
                    a[r] = *reinterpret_cast<const double2*>(kb0 + j * MOBA_D);
                    bq[r] = *reinterpret_cast<const double2*>(kb0 + j * MOBA_D + 2);
                }
            }
#pragma unroll
            for (int r = 0; r < RW; ++r) {
                double part = fma(q3, bq[r].y, fma(q2, bq[r].x, fma(q1, a[r].y, q0 * a[r].x)));
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
                const int64_t j = j0 + (int64_t)r * NW;
                if (lane == 0 && j < c) sc[j] = (part == part) ? part : -INFINITY;
            }
        }
        __syncthreads();
        // block ids of the scores, for the rank counts
        for (int64_t j = threadIdx.x; j < c; j += DEC_SEL_THREADS) sj[j] = (int32_t)j;
        __syncthreads();
        // each warp: the best kp of its slice of the blocks, by rank counts within the slice
        const int lo = (int)(c * warp / NW), hi = (int)(c * (warp + 1) / NW);
        for (int i = lo + lane; i < hi; i += 32) {
            const int rank = dec_rank(sc + lo, sj + lo, hi - lo, sc[i], i);
            if (rank < kp) {
                cs[warp * kp + rank] = sc[i];
                cj[warp * kp + rank] = i;
            }
        }
        if (lane == 0) cnt[warp] = (hi - lo < kp) ? hi - lo : kp;
        __syncthreads();
        // the head's best kp among the warps' lists, by rank counts over the compacted lists
        int n = 0;
        for (int w = 0; w < NW; ++w) {
            for (int i = threadIdx.x; i < cnt[w]; i += DEC_SEL_THREADS) {
                ms[n + i] = cs[w * kp + i];
                mj[n + i] = cj[w * kp + i];
            }
            n += cnt[w];
        }
        __syncthreads();
        for (int i = threadIdx.x; i < n; i += DEC_SEL_THREADS) {
            const int rank = dec_rank(ms, mj, n, ms[i], mj[i]);
            if (rank < kp) fj[rank] = mj[i];
        }
        __syncthreads();
        // ascending block order: winner i goes to its rank among the kp winners
        for (int i = threadIdx.x; i < kp; i += DEC_SEL_THREADS) {
            int pos = 0;
            for (int t = 0; t < kp; ++t) pos += fj[t] < fj[i];
            kept[pos] = fj[i];
        }
    } else {
        for (int j = threadIdx.x; j < npast; j += DEC_SEL_THREADS) kept[j] = j;  // every earlier block
    }
    if (p.idx_out) {
        __syncthreads();
        int32_t* orow = p.idx_out + ((int64_t)b * p.Hq + hq) * p.topk;
        for (int i = threadIdx.x; i < p.topk; i += DEC_SEL_THREADS)
            orow[i] = i < npast ? kept[i] : (i == npast ? (int32_t)c : -1);
    }
}

// ---------------------------------------------------------------- union
// grid (Hkv, B); dynamic smem: c masks. The blocks kept by any head of the group, ascending,
// with the mask of the heads that kept each, then the own block c (kept by every head).
__global__ void __launch_bounds__(DEC_UNION_THREADS) moba_decode_union_kernel(const DecodeParams p) {
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ int32_t wsum[DEC_UNION_THREADS / 32];
    const int hk = blockIdx.x, b = blockIdx.y;
    const int64_t bh = (int64_t)b * p.Hkv + hk;
    const int64_t c = p.c;
    const uint32_t all = (1u << p.G) - 1u;  // G <= 16
    int32_t* ul = p.ulist + bh * p.umax;
    uint32_t* um = p.umask + bh * p.umax;
    dec_wait_prior_grid();  // select's kept lists (and the previous step's readers of the union) are done
    dec_allow_dependents();
    if (p.full) {  // every block 0 .. c, kept by every head
        for (int64_t j = threadIdx.x; j <= c; j += DEC_UNION_THREADS) {
            ul[j] = (int32_t)j;
            um[j] = all;
        }
        if (threadIdx.x == 0) p.ucount[bh] = (int32_t)(c + 1);
        return;
    }
    uint32_t* mk = (uint32_t*)smem;  // [c]
    const int kp = p.topk - 1;
    const int kw = kp > 0 ? kp : 1;
    const int npast = (int)(c < kp ? c : kp);
    for (int64_t j = threadIdx.x; j < c; j += DEC_UNION_THREADS) mk[j] = 0u;
    __syncthreads();
    const int32_t* kept = p.kept + bh * p.G * kw;
    for (int i = threadIdx.x; i < p.G * npast; i += DEC_UNION_THREADS) {
        const int g = i / npast, r = i % npast;
        atomicOr(&mk[kept[(int64_t)g * kw + r]], 1u << g);
    }
    __syncthreads();
    // compaction in index order: thread t takes the contiguous range [t c / T, (t + 1) c / T)
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int64_t lo = c * t / DEC_UNION_THREADS, hi = c * (t + 1) / DEC_UNION_THREADS;
    int n = 0;
    for (int64_t j = lo; j < hi; ++j) n += mk[j] != 0u;
    int incl = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    int pos = incl - n;
    for (int w = 0; w < warp; ++w) pos += wsum[w];
    for (int64_t j = lo; j < hi; ++j)
        if (mk[j] != 0u) {
            ul[pos] = (int32_t)j;
            um[pos] = mk[j];
            ++pos;
        }
    if (t == DEC_UNION_THREADS - 1) {  // pos is now the number of earlier blocks in the union
        ul[pos] = (int32_t)c;
        um[pos] = all;
        p.ucount[bh] = pos + 1;
    }
}

// ---------------------------------------------------------------- attend
__device__ __forceinline__ void dec_ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void dec_ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
// D += A B, m16n8k16, A row-major bf16 (4 registers), B column-major bf16 (2), D fp32 (4)
__device__ __forceinline__ void dec_mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void dec_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void dec_wait_group() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// grid (umax * nch, Hkv, B), DEC_WARPS warps; dynamic smem DEC_ATTEND_SMEM.
// Fragments of m16n8k16 (g8 = lane / 4, t4 = lane % 4): A rows g8 and g8 + 8, columns 2 t4 (+1)
// and 2 t4 + 8 (+1); B column g8, rows 2 t4 (+1) and 2 t4 + 8 (+1); C rows g8 and g8 + 8,
// columns 2 t4 (+1). The rows are the group's heads, zero beyond G.
__global__ void __launch_bounds__(DEC_WARPS * 32, 2) moba_decode_attend_kernel(const DecodeParams p) {
    extern __shared__ __align__(16) uint8_t smem[];  // 16-byte rows for cp.async and ldmatrix
    const int hk = blockIdx.y, b = blockIdx.z;
    const int64_t bh = (int64_t)b * p.Hkv + hk;
    const int64_t u = blockIdx.x / p.nch, ch = blockIdx.x % p.nch;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g8 = lane >> 2, t4 = lane & 3;
    const int G = p.G;
    dec_allow_dependents();
    // Q as A fragments, 8 steps of 16 features (the caller's input: read before the wait)
    uint32_t qa[8][4];
    {
        const uint16_t* qb = p.q + ((int64_t)b * p.Hq + (int64_t)hk * G) * MOBA_D;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const int f = ks * 16 + 2 * t4;
            qa[ks][0] = g8 < G ? *reinterpret_cast<const uint32_t*>(qb + g8 * MOBA_D + f) : 0u;
            qa[ks][1] = g8 + 8 < G ? *reinterpret_cast<const uint32_t*>(qb + (g8 + 8) * MOBA_D + f) : 0u;
            qa[ks][2] = g8 < G ? *reinterpret_cast<const uint32_t*>(qb + g8 * MOBA_D + f + 8) : 0u;
            qa[ks][3] = g8 + 8 < G ? *reinterpret_cast<const uint32_t*>(qb + (g8 + 8) * MOBA_D + f + 8) : 0u;
        }
    }
    dec_wait_prior_grid();  // the union
    if (u >= p.ucount[bh]) return;
    const int64_t j = p.ulist[bh * p.umax + u];
    const uint32_t mask = p.umask[bh * p.umax + u];
    const int64_t bend = (j == p.c) ? p.L : (j + 1) * p.bs;  // keys [j*bs, bend)
    const int64_t k0 = j * p.bs + ch * p.chunk;
    const int64_t k1 = (k0 + p.chunk < bend) ? k0 + p.chunk : bend;
    // this warp's keys [kw0, kw1): a quarter of the chunk, in stages of 16
    const int64_t wk = p.chunk / DEC_WARPS;
    const int64_t kw0 = k0 + warp * wk;
    const int64_t kw1 = (kw0 + wk < k1) ? kw0 + wk : (k1 > kw0 ? k1 : kw0);
    const int nst = (int)((kw1 - kw0 + DEC_SKEYS - 1) / DEC_SKEYS);

    uint8_t* ring = smem + warp * (DEC_STAGES * DEC_STAGE_BYTES);
    // stage s of this warp: 16 keys of K then of V in 16-byte chunks, rows past kw1 zero-filled;
    // one commit for every stage number (empty past the last) keeps the group count uniform
    auto issue = [&](int s) {
        if (s < nst) {
            uint8_t* buf = ring + (s % DEC_STAGES) * DEC_STAGE_BYTES;
#pragma unroll 4
            for (int i = lane; i < 2 * DEC_SKEYS * 16; i += 32) {
                const int kv = i >> 8, row = (i >> 4) & 15, c16 = i & 15;
                const int64_t key = kw0 + (int64_t)s * DEC_SKEYS + row;
                const bool ok = key < kw1;
                const uint16_t* src =
                    (kv ? p.v : p.k) + (ok ? (((int64_t)b * p.Lmax + key) * p.Hkv + hk) * MOBA_D + c16 * 8 : 0);
                cp_async_16_zfill(smem_u32(buf + kv * DEC_SKEYS * DEC_ROW + row * DEC_ROW + c16 * 16), src, ok);
            }
        }
        dec_commit();
    };
    issue(0);
    issue(1);
    float o[16][4];
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
    float mu0 = -INFINITY, mu1 = -INFINITY;  // running maxima (log2 units) of rows g8, g8 + 8
    float l0 = 0.f, l1 = 0.f;                // this thread's share of the rows' sums
    const int mat = lane >> 3, r8 = lane & 7;
    for (int s = 0; s < nst; ++s) {
        issue(s + 2);
        dec_wait_group<2>();  // stage s has landed (the two newer groups may still be in flight)
        __syncwarp();
        const uint8_t* kt = ring + (s % DEC_STAGES) * DEC_STAGE_BYTES;
        const uint8_t* vt = kt + DEC_SKEYS * DEC_ROW;
        // S = Q K^T for 16 keys: n-tiles of keys 0-7 and 8-15. ldmatrix matrix `mat` of a step:
        // keys (mat / 2) * 8 .. +7, features ks * 16 + (mat % 2) * 8 .. +7
        float sa[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        {
            const uint32_t a0 = smem_u32(kt + ((mat >> 1) * 8 + r8) * DEC_ROW + (mat & 1) * 16);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                uint32_t b00, b01, b10, b11;
                dec_ldsm_x4(a0 + ks * 32, b00, b01, b10, b11);
                dec_mma(sa[0], qa[ks], b00, b01);
                dec_mma(sa[1], qa[ks], b10, b11);
            }
        }
        // scores in log2 units; keys past the warp's range masked
        const int64_t key0 = kw0 + (int64_t)s * DEC_SKEYS + 2 * t4;
        float x[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int z = 0; z < 4; ++z) {
                const bool in = key0 + nt * 8 + (z & 1) < kw1;
                x[nt][z] = in ? sa[nt][z] * p.scale_log2 : -INFINITY;
            }
        float mx0 = fmaxf(fmaxf(x[0][0], x[0][1]), fmaxf(x[1][0], x[1][1]));
        float mx1 = fmaxf(fmaxf(x[0][2], x[0][3]), fmaxf(x[1][2], x[1][3]));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        // the running maximum moves only when the row maximum passes it by more than 2^8 (so P <= 2^8
        // stays exact in range); the first stage sets it (its key 0 is a real key)
        if (mx0 > mu0 + 8.f) {
            const float f = exp2f(mu0 - mx0);  // 0 on the first stage
            l0 *= f;
#pragma unroll
            for (int nt = 0; nt < 16; ++nt) {
                o[nt][0] *= f;
                o[nt][1] *= f;
            }
            mu0 = mx0;
        }
        if (mx1 > mu1 + 8.f) {
            const float f = exp2f(mu1 - mx1);
            l1 *= f;
#pragma unroll
            for (int nt = 0; nt < 16; ++nt) {
                o[nt][2] *= f;
                o[nt][3] *= f;
            }
            mu1 = mx1;
        }
        float pr[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            pr[nt][0] = exp2f(x[nt][0] - mu0);
            pr[nt][1] = exp2f(x[nt][1] - mu0);
            pr[nt][2] = exp2f(x[nt][2] - mu1);
            pr[nt][3] = exp2f(x[nt][3] - mu1);
        }
        l0 += (pr[0][0] + pr[0][1]) + (pr[1][0] + pr[1][1]);
        l1 += (pr[0][2] + pr[0][3]) + (pr[1][2] + pr[1][3]);
        // P as the A fragment of O += P V (its 16 keys are the reduction). ldmatrix.trans matrix
        // `mat` of a step: keys (mat % 2) * 8 .. +7, features np * 16 + (mat / 2) * 8 .. +7
        const uint32_t pa[4] = {pack_bf16x2(pr[0][0], pr[0][1]), pack_bf16x2(pr[0][2], pr[0][3]),
                                pack_bf16x2(pr[1][0], pr[1][1]), pack_bf16x2(pr[1][2], pr[1][3])};
        {
            const uint32_t a0 = smem_u32(vt + ((mat & 1) * 8 + r8) * DEC_ROW + (mat >> 1) * 16);
#pragma unroll
            for (int np = 0; np < 8; ++np) {
                uint32_t v0, v1, v2, v3;
                dec_ldsm_x4_t(a0 + np * 32, v0, v1, v2, v3);
                dec_mma(o[2 * np], pa, v0, v1);
                dec_mma(o[2 * np + 1], pa, v2, v3);
            }
        }
        __syncwarp();  // every lane has read the stage before a later issue refills it
    }
    dec_wait_group<0>();
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    // combine the warps: m, l and O of every row through shared memory (over the rings)
    __syncthreads();
    float* cm = (float*)smem;                  // [DEC_WARPS][16]
    float* cl = cm + DEC_WARPS * 16;           // [DEC_WARPS][16]
    float* co = cl + DEC_WARPS * 16;           // [DEC_WARPS][16][128]
    if (t4 == 0) {
        cm[warp * 16 + g8] = nst > 0 ? mu0 : -INFINITY;
        cm[warp * 16 + g8 + 8] = nst > 0 ? mu1 : -INFINITY;
        cl[warp * 16 + g8] = l0;
        cl[warp * 16 + g8 + 8] = l1;
    }
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
        *reinterpret_cast<float2*>(co + (warp * 16 + g8) * MOBA_D + nt * 8 + 2 * t4) = make_float2(o[nt][0], o[nt][1]);
        *reinterpret_cast<float2*>(co + (warp * 16 + g8 + 8) * MOBA_D + nt * 8 + 2 * t4) =
            make_float2(o[nt][2], o[nt][3]);
    }
    __syncthreads();
    const int e = threadIdx.x;  // output feature
    for (int g = 0; g < G; ++g) {
        if (!((mask >> g) & 1u)) continue;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < DEC_WARPS; ++w) M = fmaxf(M, cm[w * 16 + g]);
        float acc = 0.f, ls = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < DEC_WARPS; ++w) {
                const float f = exp2f(cm[w * 16 + g] - M);  // 0 for a warp without keys
                acc = fmaf(f, co[(w * 16 + g) * MOBA_D + e], acc);
                ls = fmaf(f, cl[w * 16 + g], ls);
            }
        }
        float* pr = p.part + (((bh * p.umax + u) * p.nch + ch) * G + g) * DEC_PART;
        if (e == 0) {
            pr[0] = M;
            pr[1] = ls;  // 0 for an empty chunk
        }
        pr[4 + e] = acc;
    }
}

// ---------------------------------------------------------------- merge
// grid (Hq, B): out = sum_i 2^(m_i - M) o_i / sum_i 2^(m_i - M) l_i over the head's partials.
// Pass 1: the threads stride over the partials for M. Pass 2: warp w takes partials w, w + 8,
// ... (lane: features 4 lane .. 4 lane + 3); the warps' sums meet in shared memory. Both passes
// issue four partials' loads before using any.
__global__ void __launch_bounds__(DEC_MERGE_THREADS) moba_decode_merge_kernel(const DecodeParams p) {
    constexpr int NW = DEC_MERGE_THREADS / 32;
    __shared__ float red[NW];
    __shared__ float4 acc_s[NW][32];
    __shared__ float ls_s[NW];
    const int hq = blockIdx.x, b = blockIdx.y;
    const int hk = hq / p.G, g = hq % p.G;
    const int64_t bh = (int64_t)b * p.Hkv + hk;
    dec_wait_prior_grid();  // the attend partials
    const int64_t total = (int64_t)p.ucount[bh] * p.nch;  // partial i: union entry i / nch, chunk i % nch
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const float* base = p.part + bh * p.umax * p.nch * (int64_t)p.G * DEC_PART + (int64_t)g * DEC_PART;
    const uint32_t* um = p.umask + bh * p.umax;
    float M = -INFINITY;
    for (int64_t i0 = threadIdx.x; i0 < total; i0 += 4 * DEC_MERGE_THREADS) {
        float mv[4], lv[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int64_t i = i0 + (int64_t)r * DEC_MERGE_THREADS;
            lv[r] = 0.f;
            mv[r] = -INFINITY;
            if (i < total && ((um[i / p.nch] >> g) & 1u)) {
                const float* pr = base + i * p.G * DEC_PART;
                mv[r] = pr[0];
                lv[r] = pr[1];
            }
        }
#pragma unroll
        for (int r = 0; r < 4; ++r)
            if (lv[r] > 0.f) M = fmaxf(M, mv[r]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    if (lane == 0) red[warp] = M;
    __syncthreads();
    M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, red[w]);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float ls = 0.f;
    // four partials per warp and iteration, every load issued before any is used
    for (int64_t i0 = warp; i0 < total; i0 += 4 * NW) {
        float mv[4], lv[4];
        float4 ov[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int64_t i = i0 + (int64_t)r * NW;
            lv[r] = 0.f;
            mv[r] = 0.f;
            ov[r] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (i < total && ((um[i / p.nch] >> g) & 1u)) {
                const float* pr = base + i * p.G * DEC_PART;
                mv[r] = pr[0];
                lv[r] = pr[1];
                ov[r] = *reinterpret_cast<const float4*>(pr + 4 + 4 * lane);
            }
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            if (!(lv[r] > 0.f)) continue;
            const float w = exp2f(mv[r] - M);
            acc.x = fmaf(w, ov[r].x, acc.x);
            acc.y = fmaf(w, ov[r].y, acc.y);
            acc.z = fmaf(w, ov[r].z, acc.z);
            acc.w = fmaf(w, ov[r].w, acc.w);
            ls = fmaf(w, lv[r], ls);
        }
    }
    acc_s[warp][lane] = acc;
    if (lane == 0) ls_s[warp] = ls;
    __syncthreads();
    if (threadIdx.x < MOBA_D) {
        const int e = threadIdx.x;
        float a = 0.f, lt = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            const float4 v = acc_s[w][e >> 2];
            a += (e & 3) == 0 ? v.x : (e & 3) == 1 ? v.y : (e & 3) == 2 ? v.z : v.w;
            lt += ls_s[w];
        }
        p.out[((int64_t)b * p.Hq + hq) * MOBA_D + e] = __bfloat16_as_ushort(__float2bfloat16_rn(a / lt));
        if (e == 0) p.lse[(int64_t)b * p.Hq + hq] = (M + __log2f(lt)) * 0.69314718055994530942f;
    }
}
