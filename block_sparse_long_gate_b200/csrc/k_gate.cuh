// k_gate.cuh - parameter-less gating and top-k selection on CUDA cores (fp64).
//
// For query t of head hq (kv head hk = hq / G) in block c = floor(t / bs):
//   s_j = <q_t, Kbar_j> for every earlier block j < c ("MoBA project hub",
//   Step 2; "MoBA tech-report summary", section 2, score s_i), no scaling;
//   blocks after c are never candidates and c itself is always kept ("KIMI
//   MoBA" blog, section 3, causal_mask and current_block_force);
//   the k - 1 best earlier blocks are kept, higher score first and the lower
//   block index on equal scores; with c <= k - 1 all earlier blocks are kept.
// Output row: kept earlier blocks ascending, then c, then -1 padding.
//
// One thread owns one query row and keeps a sorted list of its best k - 1
// candidates in registers. Candidates arrive in ascending block order and are
// inserted only when strictly better than the current last entry, and the list
// is ordered by (score desc, block index asc), which gives the lowest-index
// tie-break. Scores are formed with fp64 fused multiply-adds
// over exact bf16 query values and the double block means.
#pragma once
#include "common.cuh"

#define GATE_ROWS 128
#define GATE_KB_ROWS 16

template <int KP>
__global__ void __launch_bounds__(GATE_ROWS) moba_gate_simt_kernel(const uint16_t* __restrict__ Q,
                                                                   const double* __restrict__ kbar,
                                                                   int32_t* __restrict__ idx, int64_t N, int Hq,
                                                                   int Hkv, int bs, int topk, int64_t nfull) {
    const int b = blockIdx.z, hq = blockIdx.y;
    const int64_t t0 = (int64_t)blockIdx.x * GATE_ROWS;
    const int64_t t = t0 + threadIdx.x;
    const int G = Hq / Hkv, hk = hq / G;
    const int kp = topk - 1;
    const bool active = t < N;
    const int64_t c = active ? t / bs : 0;
    const bool need = active && c > kp;

    __shared__ double skb[GATE_KB_ROWS][MOBA_D];

    uint32_t qr[64];
    if (need) {
        const uint4* qp = reinterpret_cast<const uint4*>(Q + (((int64_t)b * N + t) * Hq + hq) * MOBA_D);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            uint4 w = ld_nc_v4(qp + i);
            qr[4 * i + 0] = w.x;
            qr[4 * i + 1] = w.y;
            qr[4 * i + 2] = w.z;
            qr[4 * i + 3] = w.w;
        }
    }

    double ts[KP];
    int tj[KP];
#pragma unroll
    for (int i = 0; i < KP; ++i) {
        ts[i] = -INFINITY;
        tj[i] = 0x7FFFFFFF;
    }
    double thr = -INFINITY;
    int filled = 0;

    const int64_t tlast = (t0 + GATE_ROWS - 1 < N - 1) ? t0 + GATE_ROWS - 1 : N - 1;
    const int64_t cmax = tlast / bs;  // candidates of the tile: j < cmax
    const double* kb_head = kbar + ((int64_t)b * Hkv + hk) * nfull * MOBA_D;
    const bool any_need = __syncthreads_or(need);
    if (any_need) {
        for (int64_t j0 = 0; j0 < cmax; j0 += GATE_KB_ROWS) {
            __syncthreads();
            for (int i = threadIdx.x; i < GATE_KB_ROWS * MOBA_D; i += GATE_ROWS) {
                int64_t jj = j0 + i / MOBA_D;
                skb[i / MOBA_D][i % MOBA_D] = (jj < cmax) ? kb_head[jj * MOBA_D + (i % MOBA_D)] : 0.0;
            }
            __syncthreads();
            if (!need) continue;
            const int64_t jend = (j0 + GATE_KB_ROWS < c) ? j0 + GATE_KB_ROWS : c;
            for (int64_t j = j0; j < jend; ++j) {
                const double* kr = skb[j - j0];
                double s = 0.0;
#pragma unroll
                for (int e = 0; e < 64; ++e) {
                    s = fma((double)bf16lo(qr[e]), kr[2 * e], s);
                    s = fma((double)bf16hi(qr[e]), kr[2 * e + 1], s);
                }
                if (s > thr || filled < kp) {
                    double cs = s;
                    int cj = (int)j;
#pragma unroll
                    for (int i = 0; i < KP; ++i) {
                        // order: higher score first, lower block index among equal scores (a block
                        // pushed down the list may meet an equal score of a higher index)
                        if (cs > ts[i] || (cs == ts[i] && cj < tj[i])) {
                            double x = ts[i];
                            ts[i] = cs;
                            cs = x;
                            int y = tj[i];
                            tj[i] = cj;
                            cj = y;
                        }
                    }
                    if (filled < kp) ++filled;
                    if (filled == kp) {
#pragma unroll
                        for (int i = 0; i < KP; ++i)
                            if (i == kp - 1) thr = ts[i];
                    }
                }
            }
        }
    }
    if (!active) return;

    int32_t* row = idx + (((int64_t)b * Hq + hq) * N + t) * topk;
    if (!need) {  // every earlier block is kept
        for (int i = 0; i < topk; ++i) row[i] = (i < c) ? i : (i == c ? (int32_t)c : -1);
        return;
    }
    // keep the first kp entries, sort their block ids ascending
#pragma unroll
    for (int i = 0; i < KP; ++i)
        if (i >= kp) tj[i] = 0x7FFFFFFF;
#pragma unroll
    for (int a = 0; a < KP; ++a) {
#pragma unroll
        for (int i = 0; i + 1 < KP - a; ++i) {
            int lo = min(tj[i], tj[i + 1]), hi = max(tj[i], tj[i + 1]);
            tj[i] = lo;
            tj[i + 1] = hi;
        }
    }
#pragma unroll
    for (int i = 0; i < KP; ++i)
        if (i < kp) row[i] = tj[i];
    row[kp] = (int32_t)c;
}
