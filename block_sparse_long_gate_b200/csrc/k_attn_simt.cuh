// k_attn_simt.cuh - block-sparse attention on CUDA cores (fp32), one warp per
// query row. Kept as an independent cross-check of the tensor-core kernel and
// for debugging; it is not on the timed path.
//
// Row computation: logits x_u = q.k_u / sqrt(d) over the tile's key range
// (masked to u <= t on the own block), online softmax with a running maximum,
// O = sum_u exp(x_u - m) v_u / sum_u exp(x_u - m) and lse = m + ln sum exp(x_u - m)
// ("NSA vs MoBA" blog, section 1, the softmax(QK^T / sqrt(d)) V formula).
#pragma once
#include "k_attn_common.cuh"

__global__ void __launch_bounds__(128) moba_attn_simt_kernel(AttnParams a, int64_t item0) {
    const int64_t item = item0 + blockIdx.x;
    const PairInfo pi = decode_pair(a, item);
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    for (int x = 0; x < 2; ++x) {
    const TileInfo& ti = pi.t[x];
    if (ti.kind < 0) continue;
    const int64_t nrows = ti.kind == 0 ? ti.ne : ti.nt;
    for (int64_t r = w; r < nrows; r += 4) {
        int64_t t;
        int hq, slot = 0;
        if (ti.kind == 0) {
            const uint64_t e = a.entries[ti.e0 + r];
            t = entry_t(e);
            hq = entry_hq(e);
            slot = entry_slot(e);
        } else {
            t = ti.t0 + r;
            hq = ti.hq;
        }
        const int64_t khi = ti.kind == 0 ? ti.khi : t + 1;
        const uint2 qw = *reinterpret_cast<const uint2*>(a.q + (((int64_t)ti.b * a.N + t) * a.Hq + hq) * MOBA_D +
                                                         lane * 4);
        const float q0 = bf16lo(qw.x) * a.scale_log2, q1 = bf16hi(qw.x) * a.scale_log2;
        const float q2 = bf16lo(qw.y) * a.scale_log2, q3 = bf16hi(qw.y) * a.scale_log2;
        float m = -INFINITY, l = 0.f, o0 = 0.f, o1 = 0.f, o2 = 0.f, o3 = 0.f;
        for (int64_t u = ti.klo; u < khi; ++u) {
            const int64_t koff = (((int64_t)ti.b * a.N + u) * a.Hkv + ti.hk) * MOBA_D + lane * 4;
            const uint2 kw = *reinterpret_cast<const uint2*>(a.k + koff);
            float x = q0 * bf16lo(kw.x) + q1 * bf16hi(kw.x) + q2 * bf16lo(kw.y) + q3 * bf16hi(kw.y);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
            const uint2 vw = *reinterpret_cast<const uint2*>(a.v + koff);
            const float mn = fmaxf(m, x);
            const float sc = exp2f(m - mn);
            const float p = exp2f(x - mn);
            l = l * sc + p;
            o0 = o0 * sc + p * bf16lo(vw.x);
            o1 = o1 * sc + p * bf16hi(vw.x);
            o2 = o2 * sc + p * bf16lo(vw.y);
            o3 = o3 * sc + p * bf16hi(vw.y);
            m = mn;
        }
        const float inv = 1.f / l;
        const float lse = (m + log2f(l)) * 0.69314718055994530942f;
        uint2 ow;
        ow.x = pack_bf16x2(o0 * inv, o1 * inv);
        ow.y = pack_bf16x2(o2 * inv, o3 * inv);
        if (ti.kind == 0) {
            const int64_t prow = ((int64_t)ti.b * a.Hq + hq) * a.N + t;
            *reinterpret_cast<uint2*>(a.opart + (prow * a.kp + slot) * MOBA_D + lane * 4) = ow;
            if (lane == 0) a.lpart[prow * a.kp + slot] = lse;
        } else {
            *reinterpret_cast<uint2*>(a.out + (((int64_t)ti.b * a.N + t) * a.Hq + hq) * MOBA_D + lane * 4) = ow;
            if (lane == 0) a.lse[((int64_t)ti.b * a.Hq + hq) * a.N + t] = lse;
        }
    }
    }
}
