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

// grid (nfull, Hkv, B); 16 row groups x 16 threads that each read 16 bytes.
__global__ void __launch_bounds__(POOL_THREADS) moba_pool_kernel(const uint16_t* __restrict__ K,
                                                                 double* __restrict__ kbar, int64_t N,
                                                                 int Hkv, int bs, int64_t nfull, PoolAux aux) {
    const int64_t j = blockIdx.x;
    const int h = blockIdx.y, b = blockIdx.z;
    const int c16 = threadIdx.x & 15;
    const int rg = threadIdx.x >> 4;
    const int64_t rstride = (int64_t)Hkv * MOBA_D;
    const uint16_t* base = K + (((int64_t)b * N + j * bs) * Hkv + h) * MOBA_D + c16 * 8;

    double acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0;

    auto add = [&](const uint4& w) {
        acc[0] += (double)bf16lo(w.x);
        acc[1] += (double)bf16hi(w.x);
        acc[2] += (double)bf16lo(w.y);
        acc[3] += (double)bf16hi(w.y);
        acc[4] += (double)bf16lo(w.z);
        acc[5] += (double)bf16hi(w.z);
        acc[6] += (double)bf16lo(w.w);
        acc[7] += (double)bf16hi(w.w);
    };

    int u = rg;
    for (; u + 48 < bs; u += 64) {
        uint4 w0 = ld_nc_v4(base + (int64_t)u * rstride);
        uint4 w1 = ld_nc_v4(base + (int64_t)(u + 16) * rstride);
        uint4 w2 = ld_nc_v4(base + (int64_t)(u + 32) * rstride);
        uint4 w3 = ld_nc_v4(base + (int64_t)(u + 48) * rstride);
        add(w0);
        add(w1);
        add(w2);
        add(w3);
    }
    for (; u < bs; u += 16) add(ld_nc_v4(base + (int64_t)u * rstride));

    __shared__ double red[16][MOBA_D];
#pragma unroll
    for (int i = 0; i < 8; ++i) red[rg][c16 * 8 + i] = acc[i];
    __syncthreads();
    double x = 0.0;
    if (threadIdx.x < MOBA_D) {
        double s = 0.0;
#pragma unroll
        for (int g = 0; g < 16; ++g) s += red[g][threadIdx.x];
        x = s / (double)bs;
        kbar[(((int64_t)b * Hkv + h) * nfull + j) * MOBA_D + threadIdx.x] = x;
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
