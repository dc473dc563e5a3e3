// k_attn_tc.cuh - block-sparse attention on the sm_100a tensor cores.
//
// One 128-row query tile (past-block list tile, own-block tile or dense tile,
// see k_attn_common.cuh) is attended against its key range in steps of 128
// keys ("MoBA project hub", Step 3; "NSA vs MoBA" blog, section 1 formula):
//   S = Q K^T                     tcgen05.mma, A = Q (smem), B = K (smem), D in TMEM
//   P = exp2(S * log2(e)/sqrt(d) - m)   softmax warps, one thread per TMEM lane (row)
//   O += P V                      tcgen05.mma, A = P (TMEM, aliased over S), B = V (smem)
// with a running row maximum m and sum l; the result is O / l and
// lse = (m + log2 l) * ln 2.
//
// Roles (192 threads, one CTA per SM, persistent over the work items):
//   warp 0     producer: TMA loads of the K and V steps into a 3-stage ring
//   warp 1     MMA issuer (one thread) and TMEM owner
//   warps 2-5  softmax: gather the tile's Q rows (cp.async), softmax per step,
//              lazy O rescaling, epilogue (normalise, store bf16 rows + lse)
// TMEM: S0 = columns [0,128), S1 = [128,256), O = [256,384) (fp32, 128 lanes).
// The running maximum used for P only moves when the row maximum grows by more
// than 2^8 (log2 units), so O is rescaled rarely; P <= 2^8 stays exact in range.
//
// Phase rule: a parity wait for completion #k of a barrier is only sound when
// completion #k-1 is already known to have happened; each wait below names why.
//
// Every wait is bounded. A wait that reaches its limit records
// MOBA_ERR_DEVICE_TIMEOUT and raises a CTA-wide abort flag; all roles then leave
// their loops, the MMA thread waits (bounded) for its last MMAs, the producer
// for its loads in flight, and the TMEM is freed before the CTA exits.
#pragma once
#include <cuda.h>

#include "k_attn_common.cuh"

#define TC_STAGES 3
#define TC_THREADS 192
#define TC_STAGE_BYTES 65536  // K step 32 KB + V step 32 KB
#define TC_Q_BYTES 32768
#define TC_SMEM_BYTES (TC_Q_BYTES + TC_STAGES * TC_STAGE_BYTES + 1024 + 256)
#define TC_RESCALE_LOG2 8.0f

struct __align__(64) TcMaps {
    CUtensorMap k;  // 3-D view (d, Hkv, B*N) of K, box (64, 1, 128), 128-byte swizzle
    CUtensorMap v;  // same for V
};

struct TcBars {
    uint64_t kv_full[TC_STAGES];
    uint64_t kv_empty[TC_STAGES];
    uint64_t q_full;
    uint64_t s_full[2];
    uint64_t p_full[2];
    uint64_t pv_done;  // one completion per step: O holds P V of that step (used by the rescale)
    uint64_t o_full;   // one completion per tile: the tile's last P V is in O (used by the epilogue)
    uint64_t o_empty;
    uint64_t final_mma;
    uint32_t tmem_base;
    int abort_flag;
    uint32_t kv_issued[TC_STAGES];  // loads issued per stage (producer bookkeeping)
};

__device__ __forceinline__ float max3f(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Row maximum of 128 fp32 values held as 4 x 32 registers: four independent chains
// of three-input maxima, so the reduction is throughput- rather than latency-bound.
__device__ __forceinline__ float row_max128(const uint32_t (&v)[4][32]) {
    float m[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        float a = max3f(__uint_as_float(v[c][0]), __uint_as_float(v[c][1]), __uint_as_float(v[c][2]));
#pragma unroll
        for (int j = 3; j + 1 < 32; j += 2) a = max3f(a, __uint_as_float(v[c][j]), __uint_as_float(v[c][j + 1]));
        m[c] = fmaxf(a, __uint_as_float(v[c][31]));
    }
    return max3f(m[0], m[1], fmaxf(m[2], m[3]));
}

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// ---------------------------------------------------------------- packed fp32 pairs
__device__ __forceinline__ uint64_t f2pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2unpack(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// 2^x for a pair of values on the FMA pipe, to take load off the MUFU unit that
// evaluates ex2.approx (per 128-key step the exponentials would otherwise cost
// as many cycles as the two MMAs). Method: Cody-Waite style range reduction
// x = n + f with n = round(x) taken from the low mantissa bits of x + 1.5*2^23,
// f in [-1/2, 1/2]; 2^f by a degree-3 polynomial with coefficients fitted here
// for minimax relative error (7.5e-5, far below the 2^-9 rounding of P to bf16);
// 2^n is added to the exponent field with an integer add. Inputs are clamped at
// -126 so the exponent cannot underflow into the sign bit.
#define EXP2_C0 0x1.fff692p-1f
#define EXP2_C1 0x1.62f31cp-1f
#define EXP2_C2 0x1.f0de20p-3f
#define EXP2_C3 0x1.c3f704p-5f
__device__ __forceinline__ uint64_t exp2_poly2(uint64_t x2) {
    float x0, x1;
    f2unpack(x2, x0, x1);
    x2 = f2pack(fmaxf(x0, -126.f), fmaxf(x1, -126.f));
    const uint64_t t2 = fadd2(x2, f2pack(12582912.f, 12582912.f));       // round(x) in the low bits
    const uint64_t r2 = fadd2(t2, f2pack(-12582912.f, -12582912.f));     // round(x) as a float
    const uint64_t fr = ffma2(r2, f2pack(-1.f, -1.f), x2);               // x - round(x)
    uint64_t p2 = ffma2(f2pack(EXP2_C3, EXP2_C3), fr, f2pack(EXP2_C2, EXP2_C2));
    p2 = ffma2(p2, fr, f2pack(EXP2_C1, EXP2_C1));
    p2 = ffma2(p2, fr, f2pack(EXP2_C0, EXP2_C0));
    float p0, p1, t0, t1;
    f2unpack(p2, p0, p1);
    f2unpack(t2, t0, t1);
    return f2pack(__uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23)),
                  __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23)));
}
#define EXP2_POLY_PAIRS 3  // of every 8 pairs of a step, evaluated by exp2_poly2

// Bounded wait that also gives up when another role raised the abort flag.
__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    uint32_t n = 0;
    while (!mbar_try_wait(bar, parity)) {
        if (*abort_flag) return false;
        if (++n >= MOBA_SPIN_LIMIT) {
            moba_set_error(MOBA_ERR_DEVICE_TIMEOUT);
            *abort_flag = 1;
            return false;
        }
        if (n > 64) __nanosleep(64);
    }
    return true;
}

// Warp-uniform form for roles whose next instruction is a .sync.aligned tcgen05 op.
__device__ __forceinline__ bool tc_wait_warp(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    const bool ok = tc_wait(bar, parity, abort_flag);
    return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ int64_t tile_steps(const TileInfo& ti) {
    return (ti.khi - ti.klo + MOBA_KCHUNK - 1) / MOBA_KCHUNK;
}

__global__ void __launch_bounds__(TC_THREADS, 1)
    moba_attn_tc_kernel(const AttnParams a, const __grid_constant__ TcMaps maps, int64_t items) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t* sQ = smem;
    uint8_t* sKV = smem + TC_Q_BYTES;
    TcBars* bars = (TcBars*)(smem + TC_Q_BYTES + TC_STAGES * TC_STAGE_BYTES);
    volatile int* abort_flag = &bars->abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < TC_STAGES; ++s) {
            mbar_init(&bars->kv_full[s], 1);
            mbar_init(&bars->kv_empty[s], 1);
            bars->kv_issued[s] = 0;
        }
        mbar_init(&bars->q_full, 128);
        mbar_init(&bars->s_full[0], 1);
        mbar_init(&bars->s_full[1], 1);
        mbar_init(&bars->p_full[0], 128);
        mbar_init(&bars->p_full[1], 128);
        mbar_init(&bars->pv_done, 1);
        mbar_init(&bars->o_full, 1);
        mbar_init(&bars->o_empty, 128);
        mbar_init(&bars->final_mma, 1);
        bars->abort_flag = 0;
        fence_mbarrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&bars->tmem_base, 512);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&maps.k);
        prefetch_tmap(&maps.v);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            uint32_t g = 0;
            for (int64_t item = blockIdx.x; item < items && !*abort_flag; item += gridDim.x) {
                const TileInfo ti = decode_tile(a, item);
                if (ti.kind < 0) continue;
                const int64_t nst = tile_steps(ti);
                const int64_t row0 = (int64_t)ti.b * a.N + ti.klo;
                bool ok = true;
                for (int64_t i = 0; i < nst; ++i, ++g) {
                    const uint32_t s = g % TC_STAGES;
                    if (!tc_wait(&bars->kv_empty[s], ((g / TC_STAGES) & 1) ^ 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    uint8_t* st = sKV + s * TC_STAGE_BYTES;
                    mbar_arrive_expect_tx(&bars->kv_full[s], TC_STAGE_BYTES);
                    const int r = (int)(row0 + i * MOBA_KCHUNK);
                    tma_load_3d(smem_u32(st), &maps.k, &bars->kv_full[s], 0, ti.hk, r);
                    tma_load_3d(smem_u32(st + 16384), &maps.k, &bars->kv_full[s], 64, ti.hk, r);
                    tma_load_3d(smem_u32(st + 32768), &maps.v, &bars->kv_full[s], 0, ti.hk, r);
                    tma_load_3d(smem_u32(st + 49152), &maps.v, &bars->kv_full[s], 64, ti.hk, r);
                    bars->kv_issued[s] += 1;
                }
                if (!ok) break;
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc_qk = make_idesc_bf16(128, 128, 0, 0);
            const uint32_t idesc_pv = make_idesc_bf16(128, 128, 0, 1);
            const uint32_t sq = smem_u32(sQ), skv = smem_u32(sKV);
            const uint32_t tO = tmem + 256;
            uint32_t g = 0, tile_i = 0;
            bool ok = true;
            auto issue_qk = [&](uint32_t gg) {
                const uint32_t s = gg % TC_STAGES;
                const uint32_t sk = skv + s * TC_STAGE_BYTES;
                const uint32_t tS = tmem + (gg & 1) * 128;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
                    tc_mma_ss(tS, make_sdesc_sw128(sq + off, 16, 1024), make_sdesc_sw128(sk + off, 16, 1024),
                              idesc_qk, k > 0);
                }
                tc_commit(&bars->s_full[gg & 1]);
            };
            for (int64_t item = blockIdx.x; item < items && ok; item += gridDim.x) {
                const TileInfo ti = decode_tile(a, item);
                if (ti.kind < 0) continue;
                const uint32_t nst = (uint32_t)tile_steps(ti);
                if (!(ok = tc_wait(&bars->q_full, tile_i & 1, abort_flag))) break;
                tc_fence_after();
                for (uint32_t i = 0; i < nst; ++i) {
                    const uint32_t gg = g + i;
                    if (i == 0) {
                        if (!(ok = tc_wait(&bars->kv_full[gg % TC_STAGES], (gg / TC_STAGES) & 1, abort_flag))) break;
                        tc_fence_after();
                        issue_qk(gg);
                    }
                    if (i + 1 < nst) {
                        const uint32_t g1 = gg + 1;
                        if (!(ok = tc_wait(&bars->kv_full[g1 % TC_STAGES], (g1 / TC_STAGES) & 1, abort_flag))) break;
                        tc_fence_after();
                        issue_qk(g1);
                    }
                    if (!(ok = tc_wait(&bars->p_full[gg & 1], (gg >> 1) & 1, abort_flag))) break;
                    tc_fence_after();
                    if (i == 0) {
                        if (!(ok = tc_wait(&bars->o_empty, (tile_i & 1) ^ 1, abort_flag))) break;
                        tc_fence_after();
                    }
                    const uint32_t sv = skv + (gg % TC_STAGES) * TC_STAGE_BYTES + 32768;
                    const uint32_t tP = tmem + (gg & 1) * 128;
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        tc_mma_ts(tO, tP + k * 8, make_sdesc_sw128(sv + k * 2048, 16384, 1024), idesc_pv,
                                  (i > 0 || k > 0) ? 1u : 0u);
                    tc_commit(&bars->kv_empty[gg % TC_STAGES]);
                    tc_commit(&bars->pv_done);
                    if (i + 1 == nst) tc_commit(&bars->o_full);
                }
                g += nst;
                tile_i += 1;
            }
            // all MMAs issued by this thread have completed before TMEM is released
            tc_commit(&bars->final_mma);
            mbar_wait(&bars->final_mma, 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax warps
        const int r = 32 * (warp & 3) + lane;  // tile row == TMEM lane
        const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
        const uint32_t tO = tmem + 256 + lane_off;
        uint32_t g = 0, tile_i = 0;
        for (int64_t item = blockIdx.x; item < items; item += gridDim.x) {
            const TileInfo ti = decode_tile(a, item);
            if (ti.kind < 0) continue;
            const uint32_t nst = (uint32_t)tile_steps(ti);
            // row identity
            bool valid;
            int64_t t = 0;
            int hq = 0, slot = 0;
            if (ti.kind == 0) {
                valid = r < ti.ne;
                if (valid) {
                    const uint64_t e = a.entries[ti.e0 + r];
                    t = entry_t(e);
                    hq = entry_hq(e);
                    slot = entry_slot(e);
                }
            } else {
                valid = r < ti.nt;
                t = ti.t0 + r;
                hq = ti.hq;
            }
            // gather this row of Q into the swizzled tile (zero rows past the end)
            {
                const uint16_t* src = a.q + (valid ? (((int64_t)ti.b * a.N + t) * a.Hq + hq) * MOBA_D : 0);
                const uint32_t dst = smem_u32(sQ) + r * 128;
#pragma unroll
                for (int c = 0; c < 16; ++c)
                    cp_async_16_zfill(dst + (c >> 3) * 16384 + (((c & 7) ^ (r & 7)) << 4), src + c * 8, valid);
                cp_async_wait_all();
                fence_proxy_async_smem();
                mbar_arrive(&bars->q_full);
            }
            const int64_t tmask = ti.kind == 0 ? INT64_MAX : t;  // causal limit of the row
            float m_used = -INFINITY, l = 0.f;
            bool ok = true;
            for (uint32_t i = 0; i < nst; ++i) {
                const uint32_t gg = g + i;
                const uint32_t tS = tmem + (gg & 1) * 128 + lane_off;
                if (!(ok = tc_wait_warp(&bars->s_full[gg & 1], (gg >> 1) & 1, abort_flag))) break;
                tc_fence_after();
                uint32_t sr[4][32];
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, sr[c]);
                tc_wait_ld();
                const int64_t u0 = ti.klo + (int64_t)i * MOBA_KCHUNK;
                int64_t lim = ti.khi - 1 - u0;                 // last allowed column by the key range
                if (tmask - u0 < lim) lim = tmask - u0;        // and by causality
                if (lim < MOBA_KCHUNK - 1) {
#pragma unroll
                    for (int c = 0; c < 4; ++c)
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (c * 32 + j > lim) sr[c][j] = __float_as_uint(-INFINITY);
                }
                const float mx = row_max128(sr);
                const float m_new = fmaxf(m_used, mx * a.scale_log2);
                const bool need = m_new > m_used + TC_RESCALE_LOG2;
                if (__any_sync(0xffffffffu, need)) {
                    const float f = (m_used == -INFINITY) ? 0.f : ex2_approx(m_used - m_new);
                    if (i > 0) {
                        if (!(ok = tc_wait_warp(&bars->pv_done, (gg - 1) & 1, abort_flag))) break;
                        tc_fence_after();
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            uint32_t o[32];
                            tmem_ld32(tO + c * 32, o);
                            tc_wait_ld();
#pragma unroll
                            for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * f);
                            tmem_st32(tO + c * 32, o);
                        }
                        tc_wait_st();
                    }
                    l *= f;
                    m_used = m_new;
                }
                const float nm = -m_used;
                uint32_t pk[2][32];
                if (lim >= MOBA_KCHUNK - 1) {
                    // unmasked step: exponentials split between the MUFU and the FMA pipe
                    const uint64_t sc2 = f2pack(a.scale_log2, a.scale_log2), nm2 = f2pack(nm, nm);
                    uint64_t acc2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
                    for (int c = 0; c < 4; ++c)
#pragma unroll
                        for (int j = 0; j < 32; j += 2) {
                            const uint64_t x2 =
                                ffma2(f2pack(__uint_as_float(sr[c][j]), __uint_as_float(sr[c][j + 1])), sc2, nm2);
                            uint64_t p2;
                            if (((j >> 1) & 7) < EXP2_POLY_PAIRS) {
                                p2 = exp2_poly2(x2);
                            } else {
                                float x0, x1;
                                f2unpack(x2, x0, x1);
                                p2 = f2pack(ex2_approx(x0), ex2_approx(x1));
                            }
                            acc2[(j >> 1) & 3] = fadd2(acc2[(j >> 1) & 3], p2);
                            float p0, p1;
                            f2unpack(p2, p0, p1);
                            pk[c >> 1][(c & 1) * 16 + (j >> 1)] = pack_bf16x2(p0, p1);
                        }
                    const uint64_t s2 = fadd2(fadd2(acc2[0], acc2[1]), fadd2(acc2[2], acc2[3]));
                    float l0, l1;
                    f2unpack(s2, l0, l1);
                    l += l0 + l1;
                } else {
                    // masked step: MUFU only, so masked keys contribute exactly zero
                    float ls[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) ls[u] = 0.f;
#pragma unroll
                    for (int c = 0; c < 4; ++c)
#pragma unroll
                        for (int j = 0; j < 32; j += 2) {
                            const float p0 = ex2_approx(fmaf(__uint_as_float(sr[c][j]), a.scale_log2, nm));
                            const float p1 = ex2_approx(fmaf(__uint_as_float(sr[c][j + 1]), a.scale_log2, nm));
                            pk[c >> 1][(c & 1) * 16 + (j >> 1)] = pack_bf16x2(p0, p1);
                            ls[(j >> 1) & 7] += p0 + p1;
                        }
                    l += ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
                }
                tmem_st32(tS, pk[0]);
                tmem_st32(tS + 32, pk[1]);
                tc_wait_st();
                tc_fence_before();
                mbar_arrive(&bars->p_full[gg & 1]);
            }
            if (!ok) break;
            // epilogue. Waiting on pv_done here would be unsafe: the step barrier may still be two
            // phases behind (the last Q K^T was issued before the previous P V), so the tile has
            // its own barrier.
            if (!tc_wait_warp(&bars->o_full, tile_i & 1, abort_flag)) break;
            tc_fence_after();
            uint32_t ob[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(tO + c * 32, ob[c]);
            tc_wait_ld();
            tc_fence_before();
            mbar_arrive(&bars->o_empty);
            if (valid) {
                const float inv = 1.f / l;
                const float lse = (m_used + __log2f(l)) * 0.69314718055994530942f;
                uint16_t* dst;
                float* ldst;
                if (ti.kind == 0) {
                    const int64_t prow = ((int64_t)ti.b * a.Hq + hq) * a.N + t;
                    dst = a.opart + (prow * a.kp + slot) * MOBA_D;
                    ldst = a.lpart + prow * a.kp + slot;
                } else {
                    dst = a.out + (((int64_t)ti.b * a.N + t) * a.Hq + hq) * MOBA_D;
                    ldst = a.lse + ((int64_t)ti.b * a.Hq + hq) * a.N + t;
                }
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int j = 0; j < 32; j += 8) {
                        uint4 w;
                        w.x = pack_bf16x2(__uint_as_float(ob[c][j + 0]) * inv, __uint_as_float(ob[c][j + 1]) * inv);
                        w.y = pack_bf16x2(__uint_as_float(ob[c][j + 2]) * inv, __uint_as_float(ob[c][j + 3]) * inv);
                        w.z = pack_bf16x2(__uint_as_float(ob[c][j + 4]) * inv, __uint_as_float(ob[c][j + 5]) * inv);
                        w.w = pack_bf16x2(__uint_as_float(ob[c][j + 6]) * inv, __uint_as_float(ob[c][j + 7]) * inv);
                        *reinterpret_cast<uint4*>(dst + c * 32 + j) = w;
                    }
                *ldst = lse;
            }
            g += nst;
            tile_i += 1;
        }
    }

    // ---------------------------------------------------------------- teardown
    __syncthreads();
    if (warp == 0 && lane == 0 && *abort_flag) {
        // let every load already issued land before the shared memory goes away
        for (int s = 0; s < TC_STAGES; ++s) {
            const uint32_t n = bars->kv_issued[s];
            if (n > 0) mbar_wait(&bars->kv_full[s], (n - 1) & 1);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------- host side
typedef CUresult (*moba_encode_tiled_fn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                         const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                         CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                         CUtensorMapFloatOOBfill);

static moba_encode_tiled_fn moba_get_encoder() {
    static moba_encode_tiled_fn fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void* p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (moba_encode_tiled_fn)p;
    }
    return fn;
}

// K or V [B, N, Hkv, d] as a 3-D tensor (d, Hkv, B*N) with a (64, 1, 128) box.
static bool moba_make_kv_map(CUtensorMap* m, const void* base, int64_t rows, int Hkv) {
    moba_encode_tiled_fn enc = moba_get_encoder();
    if (!enc) return false;
    cuuint64_t gdim[3] = {(cuuint64_t)MOBA_D, (cuuint64_t)Hkv, (cuuint64_t)rows};
    cuuint64_t gstr[2] = {(cuuint64_t)MOBA_D * 2, (cuuint64_t)Hkv * MOBA_D * 2};
    cuuint32_t box[3] = {64, 1, MOBA_KCHUNK};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), gdim, gstr, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static int run_attention_tc(const AttnParams& a, cudaStream_t st) {
    const int64_t items = a.Pmax + a.D;
    if (items <= 0) return MOBA_OK;
    TcMaps maps;
    const int64_t rows = (int64_t)a.B * a.N;
    if (!moba_make_kv_map(&maps.k, a.k, rows, a.Hkv) || !moba_make_kv_map(&maps.v, a.v, rows, a.Hkv))
        return MOBA_ERR_CUDA;
    int dev = 0, nsm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return MOBA_ERR_CUDA;
    if (cudaFuncSetAttribute(moba_attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, TC_SMEM_BYTES) !=
        cudaSuccess)
        return MOBA_ERR_CUDA;
    const int64_t grid = items < nsm ? items : nsm;
    moba_attn_tc_kernel<<<(unsigned)grid, TC_THREADS, TC_SMEM_BYTES, st>>>(a, maps, items);
    return cudaGetLastError() == cudaSuccess ? MOBA_OK : MOBA_ERR_CUDA;
}
