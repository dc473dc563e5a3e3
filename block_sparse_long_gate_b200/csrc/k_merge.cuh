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
// every load of the row (up to 16 slots) before it uses any of them, so a row
// costs one memory latency and enough bytes are in flight to stream the
// partials at full bandwidth.
#pragma once
#include "common.cuh"
#include "k_invert.cuh"

#define MERGE_THREADS 256
#define MERGE_BATCH 16

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

// Merge of one row (b, hq, t) by one half-warp (lane i owns features 8i..8i+7).
// Every load of the row is issued before any is used: the own partial, the slot
// lse values and up to MERGE_BATCH slot partials, so a row costs one memory
// latency. The slot count comes from the row's own block when the selection was
// made by the library's gate (well formed by construction); an injected
// selection (VALIDATE) is read and checked first.
template <bool VALIDATE, int NB>
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
    uint16_t* orow = out + ((b * N + t) * Hq + hq) * MOBA_D + lane * 8;
    int p;
    if (VALIDATE) {
        p = check_row(idx + row * topk, topk, c);
        if (p < 0) {
            if (lane == 0) moba_set_error(MOBA_ERR_SELECTION);
            *reinterpret_cast<uint4*>(orow) = make_uint4(0u, 0u, 0u, 0u);
            if (lane == 0) lse[row] = __int_as_float(0x7fc00000);
            return;
        }
    } else {
        p = (int)(c < kp ? c : kp);
    }
    if (p == 0) return;  // only the own block: the partial already is the result
    const float* lrow = lpart + row * kp;
    const uint16_t* prow = opart + row * kp * MOBA_D + lane * 8;
    // issue: own partial, slot lse values (lane i: slots i, i + 16, i + 32, i + 48), first batch
    const uint4 dw = *reinterpret_cast<const uint4*>(orow);
    const float ld = lse[row];
    float lsl[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int s = lane + 16 * r;
        lsl[r] = s < p ? lrow[s] : -INFINITY;
    }
    uint4 x[NB];
#pragma unroll
    for (int u = 0; u < NB; ++u)
        if (u < p) x[u] = *reinterpret_cast<const uint4*>(prow + (int64_t)u * MOBA_D);
    // weights
    float m = fmaxf(fmaxf(ld, lsl[0]), fmaxf(lsl[1], fmaxf(lsl[2], lsl[3])));
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
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    fma8(acc, wd, dw);
    const int src_base = (threadIdx.x & 16);
    auto weight = [&](int s) {
        // weight of slot s lives in lane (s & 15), register s >> 4 of this half-warp
        const float wr = (s >> 4) == 0 ? lsl[0] : (s >> 4) == 1 ? lsl[1] : (s >> 4) == 2 ? lsl[2] : lsl[3];
        return __shfl_sync(hmask, wr, src_base + (s & 15));
    };
#pragma unroll
    for (int u = 0; u < NB; ++u) {
        const float w = weight(u);
        if (u < p) fma8(acc, w, x[u]);
    }
    for (int s0 = NB; s0 < p; s0 += NB) {  // long selections: further batches
#pragma unroll
        for (int u = 0; u < NB; ++u)
            if (s0 + u < p) x[u] = *reinterpret_cast<const uint4*>(prow + (int64_t)(s0 + u) * MOBA_D);
#pragma unroll
        for (int u = 0; u < NB; ++u) {
            const float w = weight(s0 + u);
            if (s0 + u < p) fma8(acc, w, x[u]);
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
// NB: slot partials loaded per batch (the smallest of 4, 8, 12, 16 that holds k - 1, so short
// selections keep fewer registers and more rows in flight per SM).
template <bool VALIDATE, int NB>
__global__ void __launch_bounds__(MERGE_THREADS) moba_merge_kernel(const int32_t* __restrict__ idx,
                                                                   const uint16_t* __restrict__ opart,
                                                                   const float* __restrict__ lpart, uint16_t* out,
                                                                   float* lse, int64_t N, int Hq, int bs, int topk,
                                                                   int64_t nrows) {
    const int64_t hw = (int64_t)blockIdx.x * (MERGE_THREADS / 16) + (threadIdx.x >> 4);
    const int64_t stride = (int64_t)gridDim.x * (MERGE_THREADS / 16);
    for (int64_t row = hw; row < nrows; row += stride)  // whole half-warps iterate together
        merge_row<VALIDATE, NB>(idx, opart, lpart, out, lse, N, Hq, bs, topk, row);
}
