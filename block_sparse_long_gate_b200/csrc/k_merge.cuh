// k_merge.cuh - log-sum-exp merge of a query's per-block partial results.
//
// Each kept block s of query t contributed a partial (O_s normalised by its own
// softmax sum, lse_s). The whole-selection result is ("MoBA project hub",
// Step 3, LSE-weighted fusion; "MoBA tech-report summary", section 2, step 5):
//   LSE = ln sum_s exp(lse_s),   out = sum_s exp(lse_s - LSE) O_s.
// The own-block partial is read from out / lse (written there by the attention
// kernel) and the merged result overwrites it. One warp per query row; each
// lane owns 4 of the 128 output features. HBM bound.
#pragma once
#include "common.cuh"
#include "k_invert.cuh"

__global__ void __launch_bounds__(256) moba_merge_kernel(const int32_t* __restrict__ idx,
                                                         const uint16_t* __restrict__ opart,
                                                         const float* __restrict__ lpart, uint16_t* out,
                                                         float* lse, int64_t N, int Hq, int bs, int topk,
                                                         int64_t nrows) {
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);  // (b, hq, t) flattened
    if (row >= nrows) return;
    const int64_t t = row % N;
    const int64_t bh = row / N;
    const int hq = (int)(bh % Hq);
    const int64_t b = bh / Hq;
    const int kp = topk - 1;
    const int64_t c = t / bs;
    const int32_t* sel = idx + row * topk;
    const int p = check_row(sel, topk, c);
    uint16_t* orow = out + ((b * N + t) * Hq + hq) * MOBA_D + lane * 4;
    if (p < 0) {
        if (lane == 0) moba_set_error(MOBA_ERR_SELECTION);
        *reinterpret_cast<uint2*>(orow) = make_uint2(0u, 0u);
        if (lane == 0) lse[row] = __int_as_float(0x7fc00000);
        return;
    }
    if (p == 0) return;  // only the own block: the partial is the result
    const float ld = lse[row];
    const float ls = lane < p ? lpart[row * kp + lane] : -INFINITY;  // p <= kp <= 63
    const float ls2 = lane + 32 < p ? lpart[row * kp + lane + 32] : -INFINITY;
    float m = fmaxf(fmaxf(ls, ls2), ld);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float z = (lane < p ? __expf(ls - m) : 0.f) + (lane + 32 < p ? __expf(ls2 - m) : 0.f);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    const float wd = __expf(ld - m);
    z += wd;
    const float L = m + __logf(z);
    const float inv = 1.f / z;
    const uint2 dw = *reinterpret_cast<const uint2*>(orow);
    float a0 = wd * bf16lo(dw.x), a1 = wd * bf16hi(dw.x), a2 = wd * bf16lo(dw.y), a3 = wd * bf16hi(dw.y);
    for (int s = 0; s < p; ++s) {
        const float lsv = __shfl_sync(0xffffffffu, s < 32 ? ls : ls2, s & 31);
        const float w = __expf(lsv - m);
        const uint2 pw = *reinterpret_cast<const uint2*>(opart + (row * kp + s) * MOBA_D + lane * 4);
        a0 += w * bf16lo(pw.x);
        a1 += w * bf16hi(pw.x);
        a2 += w * bf16lo(pw.y);
        a3 += w * bf16hi(pw.y);
    }
    uint2 ow;
    ow.x = pack_bf16x2(a0 * inv, a1 * inv);
    ow.y = pack_bf16x2(a2 * inv, a3 * inv);
    *reinterpret_cast<uint2*>(orow) = ow;
    if (lane == 0) lse[row] = L;
}
