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

// grid (nfull, Hkv, B); 16 row groups x 16 threads that each read 16 bytes.
__global__ void __launch_bounds__(POOL_THREADS) moba_pool_kernel(const uint16_t* __restrict__ K,
                                                                 double* __restrict__ kbar, int64_t N,
                                                                 int Hkv, int bs, int64_t nfull) {
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
    if (threadIdx.x < MOBA_D) {
        double s = 0.0;
#pragma unroll
        for (int g = 0; g < 16; ++g) s += red[g][threadIdx.x];
        kbar[(((int64_t)b * Hkv + h) * nfull + j) * MOBA_D + threadIdx.x] = s / (double)bs;
    }
}
