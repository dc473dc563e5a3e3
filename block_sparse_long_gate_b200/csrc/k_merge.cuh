// k_merge.cuh - log-sum-exp merge of a query's per-block partial results.
//
// Each kept block s of query t contributed a partial (O_s normalised by its own
// softmax sum, lse_s). The whole-selection result is ("MoBA project hub",
// Step 3, LSE-weighted fusion; "MoBA tech-report summary", section 2, step 5):
//   LSE = ln sum_s exp(lse_s),   out = sum_s exp(lse_s - LSE) O_s.
// The own-block partial is read from out / lse (written there by the attention
// kernel) and the merged result overwrites it.
//
// HBM bound: per row (slots + 1) * (2d + 4) bytes read, 2d + 4 written. A
// half-warp owns one row (16 lanes x 8 features, 16-byte accesses) and issues
// the loads of up to 8 slots before it uses any of them, so enough bytes are in
// flight to stream the partials at full bandwidth.
#pragma once
#include "common.cuh"
#include "k_invert.cuh"

#define MERGE_THREADS 256
#define MERGE_BATCH 8

__device__ __forceinline__ void fma8(float (&a)[8], float w, const uint4& x) {
    a[0] += w * bf16lo(x.x);
    a[1] += w * bf16hi(x.x);
    a[2] += w * bf16lo(x.y);
    a[3] += w * bf16hi(x.y);
    a[4] += w * bf16lo(x.z);
    a[5] += w * bf16hi(x.z);
    a[6] += w * bf16lo(x.w);
    a[7] += w * bf16hi(x.w);
}

// Merge of one row (b, hq, t) by one half-warp.
__device__ __forceinline__ void merge_row(const int32_t* __restrict__ idx, const uint16_t* __restrict__ opart,
                                          const float* __restrict__ lpart, uint16_t* out, float* lse, int64_t N,
                                          int Hq, int bs, int topk, int64_t row) {
    const int lane = threadIdx.x & 15;  // lane within the half-warp
    const unsigned hmask = (threadIdx.x & 16) ? 0xFFFF0000u : 0x0000FFFFu;
    const int64_t t = row % N;
    const int64_t bh = row / N;
    const int hq = (int)(bh % Hq);
    const int64_t b = bh / Hq;
    const int kp = topk - 1;
    const int64_t c = t / bs;
    const int32_t* sel = idx + row * topk;
    const int p = check_row(sel, topk, c);
    uint16_t* orow = out + ((b * N + t) * Hq + hq) * MOBA_D + lane * 8;
    if (p < 0) {
        if (lane == 0) moba_set_error(MOBA_ERR_SELECTION);
        *reinterpret_cast<uint4*>(orow) = make_uint4(0u, 0u, 0u, 0u);
        if (lane == 0) lse[row] = __int_as_float(0x7fc00000);
        return;
    }
    if (p == 0) return;  // only the own block: the partial already is the result
    const float ld = lse[row];
    const float* lrow = lpart + row * kp;
    // lane i holds lse of slots i, i + 16, i + 32, i + 48 (p <= 63)
    float lsl[4];
    float m = ld;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int s = lane + 16 * r;
        lsl[r] = s < p ? lrow[s] : -INFINITY;
        m = fmaxf(m, lsl[r]);
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(hmask, m, o));
    float z = 0.f;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        lsl[r] = __expf(lsl[r] - m);  // weight of slot lane + 16 r (0 beyond p)
        z += lsl[r];
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) z += __shfl_xor_sync(hmask, z, o);
    const float wd = __expf(ld - m);
    z += wd;
    const float L = m + __logf(z);
    const float inv = 1.f / z;
    float acc[8];
    {
        const uint4 dw = *reinterpret_cast<const uint4*>(orow);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.f;
        fma8(acc, wd, dw);
    }
    const uint16_t* prow = opart + row * kp * MOBA_D + lane * 8;
    const int src_base = (threadIdx.x & 16);
    for (int s0 = 0; s0 < p; s0 += MERGE_BATCH) {
        uint4 x[MERGE_BATCH];
#pragma unroll
        for (int u = 0; u < MERGE_BATCH; ++u)
            if (s0 + u < p) x[u] = *reinterpret_cast<const uint4*>(prow + (int64_t)(s0 + u) * MOBA_D);
#pragma unroll
        for (int u = 0; u < MERGE_BATCH; ++u) {
            const int s = s0 + u;
            // weight of slot s lives in lane (s & 15), register s >> 4 of this half-warp
            const float wr = (s >> 4) == 0 ? lsl[0] : (s >> 4) == 1 ? lsl[1] : (s >> 4) == 2 ? lsl[2] : lsl[3];
            const float w = __shfl_sync(hmask, wr, src_base + (s & 15));
            if (s < p) fma8(acc, w, x[u]);
        }
    }
    uint4 ow;
    ow.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
    ow.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
    ow.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
    ow.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
    *reinterpret_cast<uint4*>(orow) = ow;
    if (lane == 0) lse[row] = L;
}

// Persistent: each half-warp walks the rows with a stride of all half-warps of the grid
// (short-lived blocks of a row each left the SMs partly idle between block launches).
__global__ void __launch_bounds__(MERGE_THREADS) moba_merge_kernel(const int32_t* __restrict__ idx,
                                                                   const uint16_t* __restrict__ opart,
                                                                   const float* __restrict__ lpart, uint16_t* out,
                                                                   float* lse, int64_t N, int Hq, int bs, int topk,
                                                                   int64_t nrows) {
    const int64_t hw = (int64_t)blockIdx.x * (MERGE_THREADS / 16) + (threadIdx.x >> 4);
    const int64_t stride = (int64_t)gridDim.x * (MERGE_THREADS / 16);
    for (int64_t row = hw; row < nrows; row += stride)  // whole half-warps iterate together
        merge_row(idx, opart, lpart, out, lse, N, Hq, bs, topk, row);
}
