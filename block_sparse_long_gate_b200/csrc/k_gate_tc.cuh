// k_gate_tc.cuh - parameter-less gating and top-k on the sm_100a tensor cores.
//
// Same selection as the fp64 gate (k_gate.cuh): for query t in block c, the
// k - 1 best earlier blocks by <q_t, Kbar_j> (higher first, lower index on equal
// scores) plus c ("MoBA project hub", Step 2; "MoBA tech-report summary",
// section 2 gating and causality; "KIMI MoBA" blog, section 3 causal_mask and
// current_block_force).
//
// Scores are formed as s~_j = mu_j * sum(q) + <q, r_j>: the block centre mu_j
// times the row sum in fp32 plus a tcgen05 contraction of the exact bf16 query
// tile with the residual r_j = Kbar_j - mu_j held as two bf16 planes (hi, lo),
// accumulated in fp32 in TMEM. |s~_j - s_j| <= eps, a bound derived from the
// magnitudes involved (computed per row before its scan). One thread owns one
// query row and keeps the best k - 1 + GATE_EXTRA candidates in a sorted list of
// 32-bit keys: the score on a per-row grid of 2^18 levels over the bound
// [-R, R] of |s~| (top 18 bits) and 16383 - j (low 14 bits), so one unsigned
// compare orders two candidates by (grid level desc, block index asc) and an
// insertion is a chain of integer max / min pairs. sigma(key), the grid level's
// value, is within eps' = eps + 2 h of the exact score (h = grid step). Every
// candidate whose sigma lies within 2 eps' of the (k-1)-th best is re-scored
// exactly (fp64, the same evaluation as the fp64 gate), which decides the
// boundary exactly:
//   - candidates with sigma > T + 2 eps' are certainly kept,
//   - the exact top list needs nothing below T - 2 eps',
// where T is sigma of the (k-1)-th best key. If the kept list cannot show that
// nothing below it reaches T - 2 eps' (or a score fell off the grid), the row
// is re-scored exactly over all candidates.
//
// Roles (192 threads, persistent over 128-token tiles of one query head):
//   warp 0     TMA: Q tile (3-D map over [d, Hq, B*N]),
//              residual planes of 32 candidate blocks per step into 2 stages
//   warp 1     tcgen05.mma issuer: S (128 rows x 32 candidates, fp32) = sum over
//              the two planes and 8 K-steps of Q x plane^T, into 2 TMEM buffers
//   warps 2-5  top-k: one thread per row (TMEM lane)
// Shared memory (~74 KB) and TMEM (64 columns) are sized so that three CTAs
// share an SM and hide each other's latencies.
#pragma once
#include <cuda.h>

#include "k_attn_tc.cuh"
#include "k_pool.cuh"

#define GATE_TC_THREADS 192
#define GATE_TC_CTAS 3                    // CTAs per SM
#define GATE_EXTRA 4
#define GATE_CAND 32                      // candidate blocks per step (MMA N)
#define GATE_Q_BYTES 32768
#define GATE_PLANE_BYTES (GATE_CAND * 256)  // one bf16 plane of GATE_CAND rows x 128 features
#define GATE_STAGE_BYTES (2 * GATE_PLANE_BYTES)
#define GATE_GROUP 16                    // scores staged per TMEM load
// Per-row staging column in shared memory (stride 128 words, so row r's words sit in bank r):
// the keys of one TMEM load during the scan, then the boundary band and the sorted output.
__host__ __device__ constexpr int gate_sv_rows(int kpx) { return kpx > GATE_GROUP ? kpx : GATE_GROUP; }
__host__ __device__ constexpr int gate_tc_smem(int kpx) {
    return GATE_Q_BYTES + 2 * GATE_STAGE_BYTES + gate_sv_rows(kpx) * 128 * 4 + 1024 + 256;
}
#define GATE_TMEM_COLS 64                 // 2 score buffers of GATE_CAND columns
#define GATE_QBITS 18                     // score grid levels: 2^18
#define GATE_JBITS 14                     // block index bits of a key (MOBA_MAX_BLOCKS = 2^14)
static_assert(MOBA_MAX_BLOCKS <= (1 << GATE_JBITS), "block index does not fit the key");
static_assert(GATE_QBITS + GATE_JBITS == 32, "keys are 32-bit");

struct __align__(64) GateMaps {
    CUtensorMap q;       // (d, Hq, B*N), box (64, 1, 128)
    CUtensorMap planes;  // (d, B*Hkv*2*nfull), box (64, GATE_CAND)
};

struct GateParams {
    const uint16_t* q;
    const double* kbar;      // [B*Hkv][nfull][d]
    const float* mu;         // [B*Hkv][nfull]
    const unsigned* stats;   // [B*Hkv][2]: max |mu|, max |r| (float bits)
    int32_t* idx;
    int64_t N, nfull, tiles_per_head, ntiles;
    int B, Hq, Hkv, G, bs, topk, kp;
};

struct GateBars {
    uint64_t q_full, q_empty;
    uint64_t c_full[2], c_empty[2];
    uint64_t s_full[2], s_empty[2];
    uint64_t final_mma;
    uint32_t tmem_base;
    int abort_flag;
    uint32_t issued_q, issued_c[2];
};

struct GateTile {
    int b, hq, hk;
    int64_t t0, nt;   // tokens [t0, t0 + nt)
    int64_t ncand;    // candidate blocks [0, ncand) scored by the MMA
    int nch;          // candidate steps of GATE_CAND
};

__device__ __forceinline__ GateTile gate_tile(const GateParams& p, int64_t item) {
    GateTile g;
    const int64_t bh = item / p.tiles_per_head, m = item % p.tiles_per_head;
    g.b = (int)(bh / p.Hq);
    g.hq = (int)(bh % p.Hq);
    g.hk = g.hq / p.G;
    g.t0 = m * 128;
    g.nt = (p.N - g.t0 < 128) ? p.N - g.t0 : 128;
    const int64_t cmax = (g.t0 + g.nt - 1) / p.bs;  // own block of the last row
    g.ncand = (p.kp > 0 && cmax > p.kp) ? cmax : 0;  // no row needs scores when cmax <= k - 1
    g.nch = (int)((g.ncand + GATE_CAND - 1) / GATE_CAND);
    return g;
}

#ifdef MOBA_GATE_STATS
__device__ unsigned long long g_gate_stats[4];  // rows scored, zone re-scores, full re-scores, zone size sum
#define GATE_STAT(i, v) atomicAdd(&g_gate_stats[i], (unsigned long long)(v))
#else
#define GATE_STAT(i, v)
#endif

template <int KPX>
__global__ void __launch_bounds__(GATE_TC_THREADS, GATE_TC_CTAS)
    moba_gate_tc_kernel(const GateParams p, const __grid_constant__ GateMaps maps) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t* sQ = smem;                     // 32 KB
    uint8_t* sC = smem + GATE_Q_BYTES;      // 2 stages of GATE_STAGE_BYTES
    uint32_t* sV = (uint32_t*)(smem + GATE_Q_BYTES + 2 * GATE_STAGE_BYTES);  // [gate_sv_rows][128] staging
    GateBars* bars = (GateBars*)(smem + GATE_Q_BYTES + 2 * GATE_STAGE_BYTES + gate_sv_rows(KPX) * 128 * 4);
    volatile int* abort_flag = &bars->abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(&bars->q_full, 1);
        mbar_init(&bars->q_empty, 1 + 128);  // MMA commit + every top-k thread
        bars->issued_q = 0;
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars->c_full[i], 1);
            mbar_init(&bars->c_empty[i], 1);
            mbar_init(&bars->s_full[i], 1);
            mbar_init(&bars->s_empty[i], 128);
            bars->issued_c[i] = 0;
        }
        mbar_init(&bars->final_mma, 1);
        bars->abort_flag = 0;
        fence_mbarrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&bars->tmem_base, GATE_TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&maps.q);
        prefetch_tmap(&maps.planes);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            uint32_t ti = 0, g = 0;
            bool ok = true;
            for (int64_t item = blockIdx.x; item < p.ntiles && ok; item += gridDim.x, ++ti) {
                const GateTile gt = gate_tile(p, item);
                // completion #(ti - 1) of q_empty: #(ti - 2) was waited for the previous tile
                if (!(ok = tc_wait(&bars->q_empty, (ti & 1) ^ 1, abort_flag))) break;
                mbar_arrive_expect_tx(&bars->q_full, GATE_Q_BYTES);
                const int row = (int)((int64_t)gt.b * p.N + gt.t0);
                tma_load_3d(smem_u32(sQ), &maps.q, &bars->q_full, 0, gt.hq, row);
                tma_load_3d(smem_u32(sQ + 16384), &maps.q, &bars->q_full, 64, gt.hq, row);
                bars->issued_q += 1;
                const int64_t bh = (int64_t)gt.b * p.Hkv + gt.hk;
                for (int m = 0; m < gt.nch; ++m, ++g) {
                    const uint32_t s = g & 1;
                    if (!(ok = tc_wait(&bars->c_empty[s], ((g >> 1) & 1) ^ 1, abort_flag))) break;
                    uint8_t* st = sC + s * GATE_STAGE_BYTES;
                    mbar_arrive_expect_tx(&bars->c_full[s], GATE_STAGE_BYTES);
#pragma unroll
                    for (int pl = 0; pl < 2; ++pl) {
                        const int r = (int)((bh * 2 + pl) * p.nfull + (int64_t)m * GATE_CAND);
                        uint8_t* dst = st + pl * GATE_PLANE_BYTES;
                        tma_load_3d(smem_u32(dst), &maps.planes, &bars->c_full[s], 0, 0, r);
                        tma_load_3d(smem_u32(dst + GATE_PLANE_BYTES / 2), &maps.planes, &bars->c_full[s], 64, 0, r);
                    }
                    bars->issued_c[s] += 1;
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // The whole warp runs the loop, converged, and the elected lane (always lane 0)
        // issues each MMA and commit: the operands stay warp-uniform, which keeps the issue
        // rate when the top-k warps keep the SM sub-partition busy.
        const uint32_t idesc = make_idesc_bf16(128, GATE_CAND, 0, 0);
        const uint64_t dq = make_sdesc_sw128(smem_u32(sQ), 16, 1024);
        const uint64_t dc0 = make_sdesc_sw128(smem_u32(sC), 16, 1024);
        uint32_t ti = 0, g = 0;
        bool ok = true;
        for (int64_t item = blockIdx.x; item < p.ntiles && ok; item += gridDim.x, ++ti) {
            const GateTile gt = gate_tile(p, item);
            if (!(ok = tc_wait_warp(&bars->q_full, ti & 1, abort_flag))) break;
            tc_fence_after();
            for (int m = 0; m < gt.nch; ++m, ++g) {
                const uint32_t s = g & 1;
                if (!(ok = tc_wait_warp(&bars->c_full[s], (g >> 1) & 1, abort_flag))) break;
                // the top-k threads have read this TMEM buffer two steps ago
                if (!(ok = tc_wait_warp(&bars->s_empty[s], ((g >> 1) & 1) ^ 1, abort_flag))) break;
                tc_fence_after();
                const uint64_t dc = dc0 + (uint64_t)(s * (GATE_STAGE_BYTES >> 4));
                const uint32_t tS = tmem + s * GATE_CAND;
#pragma unroll
                for (int pl = 0; pl < 2; ++pl)
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const uint32_t qoff = ((k >> 2) * 16384 + (k & 3) * 32) >> 4;
                        const uint32_t coff =
                            (pl * GATE_PLANE_BYTES + (k >> 2) * (GATE_PLANE_BYTES / 2) + (k & 3) * 32) >> 4;
                        tc_mma_ss_w(tS, dq + qoff, dc + coff, idesc, (pl > 0 || k > 0) ? 1u : 0u);
                    }
                tc_commit_w(&bars->c_empty[s]);
                tc_commit_w(&bars->s_full[s]);
            }
            if (!ok) break;
            tc_commit_w(&bars->q_empty);  // the Q tile is no longer read by MMAs
        }
        __syncwarp();
        tc_commit_w(&bars->final_mma);
        mbar_wait(&bars->final_mma, 0);
        __syncwarp();
    } else {
        // ------------------------------------------------------------ top-k threads
        const int r = 32 * (warp & 3) + lane;
        const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
        const int kp = p.kp;
        uint32_t ti = 0, g = 0;
        for (int64_t item = blockIdx.x; item < p.ntiles; item += gridDim.x, ++ti) {
            const GateTile gt = gate_tile(p, item);
            if (!tc_wait_warp(&bars->q_full, ti & 1, abort_flag)) break;
            const bool active = r < gt.nt;
            const int64_t t = gt.t0 + r;
            const int64_t c = active ? t / p.bs : 0;
            const bool need = active && kp > 0 && c > kp;
            const uint8_t* qrow = sQ + r * 128;  // this row of the swizzled tile
            // row sum and l1 norm (exact in fp64)
            double sq64 = 0.0, l1 = 0.0;
#pragma unroll
            for (int ch = 0; ch < 16; ++ch) {
                const uint4 v = *reinterpret_cast<const uint4*>(qrow + (ch >> 3) * 16384 + (((ch & 7) ^ (r & 7)) << 4));
                const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const double a0 = (double)bf16lo(w4[u]), a1 = (double)bf16hi(w4[u]);
                    sq64 += a0 + a1;
                    l1 += fabs(a0) + fabs(a1);
                }
            }
            const float sq = (float)sq64;
            // Bounds of this row (see the file comment): |s| <= Rd, |s~ - s| <= eps <= Rd, so
            // |s~| <= Rb = Rd + eps; the key grid spans [-Rb, Rb] with step h.
            const int64_t bh = (int64_t)gt.b * p.Hkv + gt.hk;
            const double mu_max = (double)__uint_as_float(p.stats[bh * 2 + 0]);
            const double r_max = (double)__uint_as_float(p.stats[bh * 2 + 1]);
            const double Rd = mu_max * fabs(sq64) + l1 * r_max;
            const double eps = 0x1p-11 * l1 * r_max + 0x1p-20 * (mu_max * fabs(sq64) + 2.0 * Rd) + 1e-30;
            const double Rb = Rd + eps;
            const uint32_t qmax = (1u << GATE_QBITS) - 1u;
            // x = s~ * inv_h + off lands in [1, qmax]; level q = floor(x)
            const float inv_h = (float)((double)(qmax - 2u) / (2.0 * Rb));
            const float off = (float)(Rb * (double)inv_h + 1.0);
            uint32_t ts[KPX];
#pragma unroll
            for (int i = 0; i < KPX; ++i) ts[i] = 0u;  // 0: empty (every real key is >= 2^14)
            uint32_t thr = 0u;
            bool off_grid = false;
            const float* mu = p.mu + bh * p.nfull;
            bool ok = true;
            for (int m = 0; m < gt.nch; ++m, ++g) {
                const uint32_t s = g & 1;
                if (!(ok = tc_wait_warp(&bars->s_full[s], (g >> 1) & 1, abort_flag))) break;
                tc_fence_after();
                const int64_t j0 = (int64_t)m * GATE_CAND;
                const int jend = need ? (int)((c - j0 < GATE_CAND) ? c - j0 : GATE_CAND) : 0;  // candidates j < c
                const uint32_t kbase = (uint32_t)((1 << GATE_JBITS) - 1) - (uint32_t)j0;  // 16383 - j0
                uint32_t* sv = sV + r;  // this row's staged keys, stride 128 (bank = row)
#pragma unroll 1
                for (int cc = 0; cc < GATE_CAND / GATE_GROUP; ++cc) {
                    uint32_t sr[GATE_GROUP];
                    tmem_ld16(tmem + s * GATE_CAND + lane_off + cc * GATE_GROUP, sr);
                    tc_wait_ld();
                    // unrolled pass: keys, and the candidates that beat the list's last key
                    uint32_t hits = 0;
#pragma unroll
                    for (int jj = 0; jj < GATE_GROUP; ++jj) {
                        const int col = cc * GATE_GROUP + jj;
                        if (col < jend) {
                            const float v = fmaf(__ldg(mu + j0 + col), sq, __uint_as_float(sr[jj]));
                            const uint32_t lvl = __float2uint_rz(fmaf(v, inv_h, off));
                            off_grid |= (lvl - 1u) > (qmax - 1u);  // outside [1, qmax]
                            const uint32_t key = (lvl << GATE_JBITS) + (kbase - (uint32_t)col);
                            sv[jj * 128] = key;
                            if (key > thr) hits |= 1u << jj;
                        }
                    }
                    // one insertion chain in the code, entered once per hit in ascending block order
                    while (hits) {
                        const int jj = __ffs(hits) - 1;
                        hits &= hits - 1;
                        uint32_t x = sv[jj * 128];
                        if (x <= thr) continue;
#pragma unroll
                        for (int i = 0; i < KPX; ++i) {
                            const uint32_t hi = max(ts[i], x);
                            x = min(ts[i], x);
                            ts[i] = hi;
                        }
                        thr = ts[KPX - 1];
                    }
                }
                tc_fence_before();
                mbar_arrive(&bars->s_empty[s]);
            }
            if (!ok) break;
            bool overflow = false, slow = false;
            int ncert = 0, nband = 0, need_n = 0;
            if (active) {
                int32_t* orow = p.idx + (((int64_t)gt.b * p.Hq + gt.hq) * p.N + t) * p.topk;
                if (!need) {
                    if (c <= kp) {  // every earlier block is kept
                        for (int i = 0; i < p.topk; ++i) orow[i] = (i < c) ? i : (i == c ? (int32_t)c : -1);
                    } else {  // topk == 1: only the own block
                        orow[0] = (int32_t)c;
                    }
                } else {
                    // grid value of a key and its distance bound eps' to the exact score
                    const double hd = 1.0 / (double)inv_h, offd = (double)off;
                    auto sigma = [&](uint32_t key) { return ((double)(key >> GATE_JBITS) - offd) * hd; };
                    auto block_of = [&](uint32_t key) {
                        return (int)(((1u << GATE_JBITS) - 1u) - (key & ((1u << GATE_JBITS) - 1u)));
                    };
                    const double epsq = eps + 2.0 * hd;
                    uint32_t Tk = 0u;
#pragma unroll
                    for (int i = 0; i < KPX; ++i)
                        if (i == kp - 1) Tk = ts[i];
                    const double T = sigma(Tk);
                    const double lo_thr = T - 2.0 * epsq, hi_thr = T + 2.0 * epsq;
                    overflow = off_grid || ((c > KPX) && sigma(ts[KPX - 1]) >= lo_thr);
                    GATE_STAT(0, 1);
                    GATE_STAT(2, overflow ? 1 : 0);
                    // the list is sorted by key, so the certainly kept entries come first, then the band
#pragma unroll
                    for (int i = 0; i < KPX; ++i) {
                        const double si = sigma(ts[i]);
                        ncert += (ts[i] != 0u && si > hi_thr) ? 1 : 0;
                        nband += (ts[i] != 0u && si >= lo_thr && si <= hi_thr) ? 1 : 0;
                    }
                    if (overflow) ncert = 0;
                    need_n = kp - ncert;
                    // every band entry is kept when the band holds exactly the open slots (the
                    // common case): then no exact score is needed
                    slow = overflow || nband > need_n;
                    if (slow && !overflow) {  // stage the band's blocks for the exact pass
#pragma unroll
                        for (int i = 0; i < KPX; ++i)
                            if (i >= ncert && i < ncert + nband) sV[(i - ncert) * 128 + r] = (uint32_t)block_of(ts[i]);
                    }
                }
            }
            // Exact fp64 scores of the rows that need them, one warp per score: lane e
            // contracts features 4e..4e+3 and the warp sums the partials (a fixed order, so
            // equal blocks score equally). The row that owns the candidates keeps the best
            // need_n by (exact score desc, block index asc).
            double es[KPX];
            int ej[KPX];
            int ne = 0;
            {
                const double* kbh = p.kbar + ((int64_t)gt.b * p.Hkv + gt.hk) * p.nfull * MOBA_D;
                __syncwarp();  // the staged bands are visible to the whole warp
                unsigned pend = __ballot_sync(0xffffffffu, slow);
                while (pend) {
                    const int L = __ffs(pend) - 1;
                    pend &= pend - 1;
                    const int rL = 32 * (warp & 3) + L;
                    const bool ovL = __shfl_sync(0xffffffffu, overflow, L);
                    const int nL = ovL ? (int)__shfl_sync(0xffffffffu, (int)c, L) : __shfl_sync(0xffffffffu, nband, L);
                    const int needL = __shfl_sync(0xffffffffu, need_n, L);
                    // this lane's four features of row rL (swizzled tile: 16-byte chunk lane / 2)
                    const uint2 qv = *reinterpret_cast<const uint2*>(
                        sQ + rL * 128 + ((lane >> 1) >> 3) * 16384 + ((((lane >> 1) & 7) ^ (rL & 7)) << 4) + (lane & 1) * 8);
                    const double q0 = (double)bf16lo(qv.x), q1 = (double)bf16hi(qv.x);
                    const double q2 = (double)bf16lo(qv.y), q3 = (double)bf16hi(qv.y);
#pragma unroll 1
                    for (int u = 0; u < nL; ++u) {
                        const int jz = ovL ? u : (int)sV[u * 128 + rL];
                        const double* kr = kbh + (int64_t)jz * MOBA_D + 4 * lane;
                        const double2 a = __ldg(reinterpret_cast<const double2*>(kr));
                        const double2 b2 = __ldg(reinterpret_cast<const double2*>(kr + 2));
                        double e = q0 * a.x;
                        e = fma(q1, a.y, e);
                        e = fma(q2, b2.x, e);
                        e = fma(q3, b2.y, e);
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) e += __shfl_xor_sync(0xffffffffu, e, o);
                        GATE_STAT(3, lane == 0 ? 1 : 0);
                        if (lane == L) {
                            int pos = ne;
                            while (pos > 0 && (e > es[pos - 1] || (e == es[pos - 1] && jz < ej[pos - 1]))) --pos;
                            if (pos < needL) {
                                const int last = ne < needL ? ne : needL - 1;
                                for (int z = last; z > pos; --z) {
                                    es[z] = es[z - 1];
                                    ej[z] = ej[z - 1];
                                }
                                es[pos] = e;
                                ej[pos] = jz;
                                if (ne < needL) ++ne;
                            }
                        }
                    }
                }
                __syncwarp();  // every lane has read the staged bands before they are overwritten
            }
            if (need) {
                // kept blocks in ascending order: insertion sort in this row's staging column
                int32_t* orow = p.idx + (((int64_t)gt.b * p.Hq + gt.hq) * p.N + t) * p.topk;
                uint32_t* srow = sV + r;
                int n = 0;
                auto put = [&](uint32_t v) {
                    int u = n++;
                    while (u > 0 && srow[(u - 1) * 128] > v) {
                        srow[u * 128] = srow[(u - 1) * 128];
                        --u;
                    }
                    srow[u * 128] = v;
                };
                const int nfirst = slow ? ncert : kp;  // leading list entries that are kept
#pragma unroll
                for (int i = 0; i < KPX; ++i)
                    if (i < nfirst) put((uint32_t)(((1u << GATE_JBITS) - 1u) - (ts[i] & ((1u << GATE_JBITS) - 1u))));
                for (int u = 0; u < ne; ++u) put((uint32_t)ej[u]);
                for (int i2 = 0; i2 < kp; ++i2) orow[i2] = (int32_t)srow[i2 * 128];
                orow[kp] = (int32_t)c;
            }
            mbar_arrive(&bars->q_empty);  // this row of the Q tile is no longer read
        }
    }

    __syncthreads();
    if (warp == 0 && lane == 0 && *abort_flag) {
        if (bars->issued_q) mbar_wait(&bars->q_full, (bars->issued_q - 1) & 1);
        for (int i = 0; i < 2; ++i)
            if (bars->issued_c[i]) mbar_wait(&bars->c_full[i], (bars->issued_c[i] - 1) & 1);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, GATE_TMEM_COLS);
}

// ---------------------------------------------------------------- host side
static bool moba_make_2d_map(CUtensorMap* m, const void* base, int64_t rows) {
    moba_encode_tiled_fn enc = moba_get_encoder();
    if (!enc) return false;
    cuuint64_t gdim[3] = {(cuuint64_t)MOBA_D, 1, (cuuint64_t)rows};
    cuuint64_t gstr[2] = {(cuuint64_t)MOBA_D * 2, (cuuint64_t)MOBA_D * 2};
    cuuint32_t box[3] = {64, 1, GATE_CAND};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), gdim, gstr, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int KPX>
static int launch_gate_tc(const GateParams& gp, const GateMaps& maps, int grid, cudaStream_t st) {
    if (cudaFuncSetAttribute(moba_gate_tc_kernel<KPX>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             gate_tc_smem(KPX)) != cudaSuccess)
        return MOBA_ERR_CUDA;
    moba_gate_tc_kernel<KPX><<<grid, GATE_TC_THREADS, gate_tc_smem(KPX), st>>>(gp, maps);
    const cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) {
        cudaGetLastError();
        (void)cudaPeekAtLastError();
        moba_note_cuda_error(err);
        return MOBA_ERR_CUDA;
    }
    return MOBA_OK;
}

static int run_gate_tc(const GateParams& gp, const uint16_t* planes, cudaStream_t st) {
    GateMaps maps;
    if (!moba_make_kv_map(&maps.q, gp.q, (int64_t)gp.B * gp.N, gp.Hq)) return MOBA_ERR_CUDA;
    if (!moba_make_2d_map(&maps.planes, planes, (int64_t)gp.B * gp.Hkv * 2 * gp.nfull)) return MOBA_ERR_CUDA;
    int dev = 0, nsm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return MOBA_ERR_CUDA;
    const int grid = (int)(gp.ntiles < GATE_TC_CTAS * nsm ? gp.ntiles : GATE_TC_CTAS * nsm);
    if (gp.kp + GATE_EXTRA <= 8) return launch_gate_tc<8>(gp, maps, grid, st);
    if (gp.kp + GATE_EXTRA <= 16) return launch_gate_tc<16>(gp, maps, grid, st);
    if (gp.kp + GATE_EXTRA <= 24) return launch_gate_tc<24>(gp, maps, grid, st);
    if (gp.kp + GATE_EXTRA <= 40) return launch_gate_tc<40>(gp, maps, grid, st);
    return launch_gate_tc<72>(gp, maps, grid, st);
}
