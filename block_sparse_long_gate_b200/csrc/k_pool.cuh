// k_pool.cuh - block mean pooling of the keys.
//
// Kbar[b, h, j, :] = (1 / block_size) * sum of K[b, u, h, :] over the keys u of
// full block j ("KIMI MoBA" blog, section 3, score_pooling = mean; "MoBA project
// hub", Step 2). Only full blocks are pooled: a query's past blocks are always
// full, and the last (possibly partial) block is never a past block.
//
// Each bf16 key is added in double precision. A sum of up to 2^21 bf16 values
// of one block is exact in double for the value ranges of the workloads, so the
// mean carries a single rounding (the division) and the gate sees the same
// block representatives as an exact evaluation would.
//
// Variants ("KIMI MoBA" blog, section 6: try max or weighted pooling): the
// feature-wise maximum over the block's keys (exact), or the weighted mean
// sum_p w[p] K[jB + p] / sum_p w[p] with one fp32 weight per position inside a
// block (products and sums in double).
//
// Streaming reduction, HBM bound: 2 * block_size * d bytes read per (b, h, j).
#pragma once
#include "common.cuh"

#define POOL_THREADS 256

// Extra outputs for the tensor-core gate (all null when only Kbar is wanted):
// each block mean is written as a centre mu_j (fp32, the mean over the d
// features) plus a residual r_j = Kbar_j - mu_j split into two bf16 planes
// (hi = bf16(r), lo = bf16(r - hi)), so that <q, Kbar_j> = mu_j * sum(q) + <q, r_j>
// with the cancellation-prone part small. head_stats[(b*Hkv+h)*2 + {0,1}] receive
// max_j |mu_j| and max_{j,d} |r_jd| (float bits, non-negative, so integer atomicMax
// orders them) for the gate's error bound.
struct PoolAux {
    uint16_t* planes;       // bf16 [B*Hkv][2][nfull][d]
    float* mu;              // fp32 [B*Hkv][nfull]
    unsigned* head_stats;   // [B*Hkv][2], zeroed before the launch
};

// Pooling of a block: 0 mean, 1 feature-wise max, 2 weighted mean with weights w[0, bs).
// j0 / rows: the grid pools blocks j0 + blockIdx.x into rows of a summary buffer with `rows`
// rows per (b, kv head) (a KV cache pools only the blocks that became full; rows = 0 means nfull).
struct PoolMode {
    int mode;
    const float* w;
    int64_t j0 = 0;
    int64_t rows = 0;
};

// grid (nfull, Hkv, B); 16 row groups x 16 threads that each read 16 bytes.
__global__ void __launch_bounds__(POOL_THREADS) moba_pool_kernel(const uint16_t* __restrict__ K,
                                                                 double* __restrict__ kbar, int64_t N,
                                                                 int Hkv, int bs, int64_t nfull, PoolAux aux,
                                                                 PoolMode pm) {
    const int64_t j = pm.j0 + blockIdx.x;
    const int64_t krows = pm.rows > 0 ? pm.rows : nfull;
    const int h = blockIdx.y, b = blockIdx.z;
    const int c16 = threadIdx.x & 15;
    const int rg = threadIdx.x >> 4;
    const int64_t rstride = (int64_t)Hkv * MOBA_D;
    const uint16_t* base = K + (((int64_t)b * N + j * bs) * Hkv + h) * MOBA_D + c16 * 8;

    const bool is_max = pm.mode == 1, is_w = pm.mode == 2;
    double acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = is_max ? -INFINITY : 0.0;

    auto add = [&](const uint4& w, double wt) {
        const float f[8] = {bf16lo(w.x), bf16hi(w.x), bf16lo(w.y), bf16hi(w.y),
                            bf16lo(w.z), bf16hi(w.z), bf16lo(w.w), bf16hi(w.w)};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (is_max) acc[i] = fmax(acc[i], (double)f[i]);
            else if (is_w) acc[i] = fma(wt, (double)f[i], acc[i]);
            else acc[i] += (double)f[i];
        }
    };
    auto wt_at = [&](int u) { return is_w ? (double)__ldg(pm.w + u) : 1.0; };

    int u = rg;
    for (; u + 48 < bs; u += 64) {
        uint4 w0 = ld_nc_v4(base + (int64_t)u * rstride);
        uint4 w1 = ld_nc_v4(base + (int64_t)(u + 16) * rstride);
        uint4 w2 = ld_nc_v4(base + (int64_t)(u + 32) * rstride);
        uint4 w3 = ld_nc_v4(base + (int64_t)(u + 48) * rstride);
        add(w0, wt_at(u));
        add(w1, wt_at(u + 16));
        add(w2, wt_at(u + 32));
        add(w3, wt_at(u + 48));
    }
    for (; u < bs; u += 16) add(ld_nc_v4(base + (int64_t)u * rstride), wt_at(u));

    __shared__ double red[16][MOBA_D];
    __shared__ double wred[POOL_THREADS / 32];
    __shared__ int wbad;
#pragma unroll
    for (int i = 0; i < 8; ++i) red[rg][c16 * 8 + i] = acc[i];
    double wsum = (double)bs;
    if (is_w) {  // sum of the weights (and a check that none is negative)
        double sw = 0.0;
        int bad = 0;
        for (int p = threadIdx.x; p < bs; p += POOL_THREADS) {
            const float wp = __ldg(pm.w + p);
            sw += (double)wp;
            bad |= !(wp >= 0.f);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sw += __shfl_xor_sync(0xffffffffu, sw, o);
        bad = __any_sync(0xffffffffu, bad);
        if (threadIdx.x == 0) wbad = 0;
        __syncthreads();
        if ((threadIdx.x & 31) == 0) {
            wred[threadIdx.x >> 5] = sw;
            if (bad) wbad = 1;
        }
    }
    __syncthreads();
    if (is_w) {
        wsum = 0.0;
#pragma unroll
        for (int i = 0; i < POOL_THREADS / 32; ++i) wsum += wred[i];
        if (threadIdx.x == 0 && (wbad || !(wsum > 0.0))) moba_set_error(MOBA_ERR_VALUE);
    }
    double x = 0.0;
    if (threadIdx.x < MOBA_D) {
        double s = is_max ? -INFINITY : 0.0;
#pragma unroll
        for (int g = 0; g < 16; ++g) s = is_max ? fmax(s, red[g][threadIdx.x]) : s + red[g][threadIdx.x];
        x = is_max ? s : s / wsum;
        kbar[(((int64_t)b * Hkv + h) * krows + j) * MOBA_D + threadIdx.x] = x;
    }
    if (aux.planes == nullptr) return;
    // centre and residual planes (threads 0..127 own one feature each)
    __shared__ double red2[4];
    __shared__ float fred[4];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    double sx = x;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sx += __shfl_xor_sync(0xffffffffu, sx, o);
    if (lane == 0 && w < 4) red2[w] = sx;
    __syncthreads();
    const float mu = (float)((red2[0] + red2[1] + red2[2] + red2[3]) / (double)MOBA_D);
    const int64_t bh = (int64_t)b * Hkv + h;
    float ar = 0.f;
    if (threadIdx.x < MOBA_D) {
        const double r = x - (double)mu;
        const __nv_bfloat16 hi = __float2bfloat16_rn((float)r);
        const __nv_bfloat16 lo = __float2bfloat16_rn((float)(r - (double)__bfloat162float(hi)));
        aux.planes[((bh * 2 + 0) * nfull + j) * MOBA_D + threadIdx.x] = __bfloat16_as_ushort(hi);
        aux.planes[((bh * 2 + 1) * nfull + j) * MOBA_D + threadIdx.x] = __bfloat16_as_ushort(lo);
        ar = (float)fabs(r) * (1.0f + 1.0f / 1024.0f);  // rounded up: a bound on |r|
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ar = fmaxf(ar, __shfl_xor_sync(0xffffffffu, ar, o));
    if (lane == 0 && w < 4) fred[w] = ar;
    __syncthreads();
    if (threadIdx.x == 0) {
        const float rm = fmaxf(fmaxf(fred[0], fred[1]), fmaxf(fred[2], fred[3]));
        aux.mu[bh * nfull + j] = mu;
        atomicMax(&aux.head_stats[bh * 2 + 0], __float_as_uint(fabsf(mu)));
        atomicMax(&aux.head_stats[bh * 2 + 1], __float_as_uint(rm));
    }
}
