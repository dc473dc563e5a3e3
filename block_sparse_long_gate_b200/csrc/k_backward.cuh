// k_backward.cuh - the backward of the MoBA attention on the sm_100a tensor cores.
//
// With the selection fixed (the top-k choice is discrete, so the block summaries get
// no gradient), for the loss sum_t <dO_t, out_t> ("MoBA tech-report summary",
// section 3 trains with MoBA; gradients of softmax(q k^T / sqrt(d)) v):
//   P_tu = exp(q_t.k_u / sqrt(d) - lse_t),  D_t = <dO_t, out_t>
//   dS_tu = P_tu (<dO_t, v_u> - D_t)
//   dQ_t = sum_u dS_tu k_u / sqrt(d),  dK_u = sum_t dS_tu q_t / sqrt(d),  dV_u = sum_t P_tu dO_t
//
// Work item = one 128-key step of one key block j of one (b, kv head): the CTA
// keeps dK and dV of those keys in TMEM and walks every query that reads them:
// the past-block list of j (the forward's inverted selection) and the causal
// own-block queries of j of every query head of the group. Per 128-row query tile
// (tcgen05, fp32 accumulation; keys on the TMEM lanes):
//   S^T  = K Q^T          SS (K, Q K-major)                  -> TMEM S
//   dP^T = V dO^T         SS (V, dO K-major)                 -> TMEM dP
//   P^T, dS^T  by the 256 threads (two per key, each half of the queries), bf16
//              into TMEM over S / dP, dS also into shared memory (the A operand
//              of dQ, query-major)
//   dV += P^T dO          TS (A from TMEM, dO MN-major)
//   dK += dS^T Q          TS (A from TMEM, Q MN-major)
//   dQ  = dS K            SS (dS MN-major, K MN-major)       -> TMEM S
//   dQ rows (thread = query) are added to an fp32 accumulator: each thread
//   stages its 512-byte row in shared memory (over the Q and dO tiles, free once
//   the products are done) and adds it with one bulk reduction
//   (cp.reduce.async.bulk .add.f32), which the L2 performs about three times as
//   fast as per-thread vector atomics; a last kernel scales and rounds to bf16.
// Roles are not split: two warpgroups gather, wait, compute and reduce in turn,
// warps w and w + 4 sharing TMEM lanes 32 (w % 4) .. + 31 (a key, or a query for
// dQ) and splitting the columns, so each scheduler has two warps to switch between.
#pragma once
#include <cuda.h>

#include "k_attn_tc.cuh"

#define BWD_THREADS 256
#define BWD_TILE_BYTES 32768  // 128 rows x 128 d x bf16
#define BWD_SMEM_BYTES (5 * BWD_TILE_BYTES + 2048 + 1024)
#define BWD_DQ_STRIDE 528  // bytes per staged dQ row: 512 + 16, so 8 threads storing 16 bytes each hit distinct banks
static_assert(128 * BWD_DQ_STRIDE <= 3 * BWD_TILE_BYTES, "the dQ staging must fit over the Q, dO and dS tiles");

struct BwdParams {
    const uint16_t* q;    // [B, N, Hq, d]
    const uint16_t* dout;
    const float* lse;     // [B, Hq, N] natural log
    const float* Dvec;    // [B, Hq, N]
    uint16_t* dk;         // [B, N, Hkv, d]
    uint16_t* dv;
    float* dq_acc;        // [B, N, Hq, d] fp32, zeroed
    const uint64_t* entries;
    const int64_t* segoff;  // list l spans entries [segoff[l*nch], segoff[(l+1)*nch])
    int* counter;           // work counter, zeroed
    int64_t N, nblk, nch, mb, items;
    int B, Hq, Hkv, G, bs;
    float scale_log2;       // log2(e) / sqrt(d)
    float scale;            // 1 / sqrt(d)
};

struct BwdBars {
    uint64_t kv_full;
    uint64_t mma;
    uint32_t tmem_base;
    int item;
    int abort_flag;
};

#ifdef MOBA_BWD_DEBUG
__device__ long long g_bwd_dbg[8];  // wait id, item, tile, phase of the first wait that gave up
#define BWD_NOTE(id, it, qt, ph)                                                                     \
    if (atomicCAS((unsigned long long*)&g_bwd_dbg[0], 0ull, (unsigned long long)(id)) == 0ull) {  \
        g_bwd_dbg[1] = (it);                                                                         \
        g_bwd_dbg[2] = (qt);                                                                         \
        g_bwd_dbg[3] = (ph);                                                                         \
    }
#else
#define BWD_NOTE(id, it, qt, ph)
#endif

// D_t = <dO_t, out_t> in fp32, one half-warp per row (b, hq, t)
__global__ void __launch_bounds__(256) moba_bwd_prep_kernel(const uint16_t* __restrict__ out,
                                                            const uint16_t* __restrict__ dout, float* __restrict__ D,
                                                            int64_t N, int Hq, int64_t nrows) {
    const int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 4;
    const int lane = threadIdx.x & 15;
    const unsigned hmask = (threadIdx.x & 16) ? 0xFFFF0000u : 0x0000FFFFu;
    if (row >= nrows) return;  // whole half-warps leave together
    const int64_t t = row % N, bh = row / N;
    const int hq = (int)(bh % Hq);
    const int64_t b = bh / Hq;
    const int64_t off = ((b * N + t) * Hq + hq) * MOBA_D + lane * 8;
    const uint4 o = ld_nc_v4(out + off), g = ld_nc_v4(dout + off);
    float s = bf16lo(o.x) * bf16lo(g.x) + bf16hi(o.x) * bf16hi(g.x) + bf16lo(o.y) * bf16lo(g.y) +
              bf16hi(o.y) * bf16hi(g.y) + bf16lo(o.z) * bf16lo(g.z) + bf16hi(o.z) * bf16hi(g.z) +
              bf16lo(o.w) * bf16lo(g.w) + bf16hi(o.w) * bf16hi(g.w);
#pragma unroll
    for (int o2 = 8; o2 > 0; o2 >>= 1) s += __shfl_xor_sync(hmask, s, o2);
    if (lane == 0) D[row] = s;
}

// dq = bf16(dq_acc / sqrt(d))
__global__ void __launch_bounds__(256) moba_bwd_dq_kernel(const float* __restrict__ acc, uint16_t* __restrict__ dq,
                                                          float scale, int64_t n4) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n4) return;
    const float4 a = reinterpret_cast<const float4*>(acc)[i];
    uint2 w;
    w.x = pack_bf16x2(a.x * scale, a.y * scale);
    w.y = pack_bf16x2(a.z * scale, a.w * scale);
    reinterpret_cast<uint2*>(dq)[i] = w;
}

// dst[0 .. bytes/4) += src[...] (fp32), read from shared memory by the bulk-copy unit; bytes is a
// multiple of 16 and both addresses are 16-byte aligned. Completion is tracked by bulk groups.
__device__ __forceinline__ void bulk_reduce_add_f32(float* dst, uint32_t src_smem, uint32_t bytes) {
    asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;" ::"l"(dst),
                 "r"(src_smem), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// this thread's bulk operations have read their shared-memory sources
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// this thread's bulk operations are complete
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__global__ void __launch_bounds__(BWD_THREADS, 1)
    moba_bwd_kernel(const BwdParams p, const __grid_constant__ TcMaps maps) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    if (smem_u32(smem_raw) & 1023) {
        if (threadIdx.x == 0) moba_set_error(MOBA_ERR_UNSUPPORTED);
        return;
    }
    uint8_t* sK = smem_raw;
    uint8_t* sV = sK + BWD_TILE_BYTES;
    uint8_t* sQ = sV + BWD_TILE_BYTES;
    uint8_t* sG = sQ + BWD_TILE_BYTES;   // dO tile
    uint8_t* sS = sG + BWD_TILE_BYTES;   // dS tile, query-major (A operand of dQ)
    float* sL = (float*)(sS + BWD_TILE_BYTES);  // lse (log2 units) of the tile's rows, +inf if empty
    float* sD = sL + 128;                       // D of the tile's rows
    int64_t* sRow = (int64_t*)(sD + 128);       // dq_acc row offset of each query row, -1 if empty
    BwdBars* bars = (BwdBars*)(smem_raw + 5 * BWD_TILE_BYTES + 2048);
    const int warp = threadIdx.x >> 5;
    const int r = threadIdx.x & 127;  // TMEM lane: a key (S^T, dP^T, dK, dV) or a query (dQ)
    const int h = threadIdx.x >> 7;   // which half of the columns this thread takes

    if (threadIdx.x == 0) {
        mbar_init(&bars->kv_full, 1);
        mbar_init(&bars->mma, 1);
        bars->abort_flag = 0;
        fence_mbarrier_init();
        prefetch_tmap(&maps.k);
        prefetch_tmap(&maps.v);
    }
    if (warp == 0) {
        tmem_alloc(&bars->tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const uint32_t tS = tmem, tP = tmem + 128, tK = tmem + 256, tV = tmem + 384;
    const uint32_t idesc_ss = make_idesc_bf16(128, 128, 0, 0);   // both K-major
    const uint32_t idesc_ts = make_idesc_bf16(128, 128, 0, 1);   // A in TMEM, B MN-major
    const uint32_t idesc_dq = make_idesc_bf16(128, 128, 1, 1);   // A and B MN-major
    const uint64_t dK_k = make_sdesc_sw128(smem_u32(sK), 16, 1024);
    const uint64_t dV_k = make_sdesc_sw128(smem_u32(sV), 16, 1024);
    const uint64_t dQ_k = make_sdesc_sw128(smem_u32(sQ), 16, 1024);
    const uint64_t dG_k = make_sdesc_sw128(smem_u32(sG), 16, 1024);
    const uint64_t dQ_mn = make_sdesc_sw128(smem_u32(sQ), 16384, 1024);
    const uint64_t dG_mn = make_sdesc_sw128(smem_u32(sG), 16384, 1024);
    const uint64_t dK_mn = make_sdesc_sw128(smem_u32(sK), 16384, 1024);
    const uint64_t dS_mn = make_sdesc_sw128(smem_u32(sS), 16384, 1024);
    uint32_t kv_phase = 0, mma_phase = 0;
    bool ok = true;
    volatile int* abort_flag = &bars->abort_flag;

    for (;;) {
        if (threadIdx.x == 0) bars->item = atomicAdd(p.counter, 1);
        __syncthreads();
        const int64_t item = bars->item;
        __syncthreads();  // every thread has read the item before thread 0 may take the next one
        if (item >= p.items || !ok) break;
        const int64_t l = item / p.mb, step = item % p.mb;
        const int64_t j = l % p.nblk;
        const int hk = (int)((l / p.nblk) % p.Hkv);
        const int b = (int)(l / (p.nblk * p.Hkv));
        const int64_t bend = (j * p.bs + p.bs < p.N) ? j * p.bs + p.bs : p.N;
        const int64_t u0 = j * p.bs + step * MOBA_KCHUNK;
        if (u0 >= bend) continue;  // a step past the end of a short block: no keys
        const int ku = (int)((bend - u0 < MOBA_KCHUNK) ? bend - u0 : MOBA_KCHUNK);

        // K and V of the step (the TMA zero-fills rows past the tensor; rows past the block are masked)
        if (threadIdx.x == 0) {
            mbar_arrive_expect_tx(&bars->kv_full, 2 * BWD_TILE_BYTES);
            const int row = (int)((int64_t)b * p.N + u0);
            tma_load_3d(smem_u32(sK), &maps.k, &bars->kv_full, 0, hk, row);
            tma_load_3d(smem_u32(sK + 16384), &maps.k, &bars->kv_full, 64, hk, row);
            tma_load_3d(smem_u32(sV), &maps.v, &bars->kv_full, 0, hk, row);
            tma_load_3d(smem_u32(sV + 16384), &maps.v, &bars->kv_full, 64, hk, row);
        }
        // wall-clock bounded (a wait that gives up records MOBA_ERR_DEVICE_TIMEOUT and aborts the CTA)
        ok = tc_wait(&bars->kv_full, kv_phase & 1, abort_flag);
        if (!ok) BWD_NOTE(1, item, -1, kv_phase);
        if (!(ok = __syncthreads_and(ok))) break;  // the whole CTA gives up together
        ++kv_phase;

        // query tiles: the past list of j, then the own-block rows of every head of the group
        const int64_t e_lo = p.segoff[l * p.nch], e_hi = p.segoff[(l + 1) * p.nch];
        const int64_t n_past = (e_hi - e_lo + 127) / 128;
        const int64_t n_diag_per_head = (bend - u0 + 127) / 128;
        const int64_t n_tiles = n_past + n_diag_per_head * p.G;
        for (int64_t qt = 0; qt < n_tiles && ok; ++qt) {
            const bool past = qt < n_past;
            // ---- gather this tile's query rows (thread r gathers row r)
            bool valid;
            int64_t t = 0;
            int hq = 0;
            int64_t tdiag0 = 0;  // first query of a diagonal tile
            if (past) {
                const int64_t e = e_lo + qt * 128 + r;
                valid = e < e_hi;
                if (valid) {
                    const uint64_t en = p.entries[e];
                    t = entry_t(en);
                    hq = entry_hq(en);
                }
            } else {
                const int64_t dq_i = qt - n_past;
                hq = hk * p.G + (int)(dq_i / n_diag_per_head);
                tdiag0 = u0 + (dq_i % n_diag_per_head) * 128;
                t = tdiag0 + r;
                valid = t < bend;
            }
            const int64_t qrow = ((int64_t)b * p.N + t) * p.Hq + hq;  // row of q / dO / dq_acc
            const int64_t lrow = ((int64_t)b * p.Hq + hq) * p.N + t;  // row of lse / D
            {
                const uint16_t* srcq = p.q + (valid ? qrow * MOBA_D : 0);
                const uint16_t* srcg = p.dout + (valid ? qrow * MOBA_D : 0);
                const uint32_t dq_s = smem_u32(sQ) + r * 128, dg_s = smem_u32(sG) + r * 128;
#pragma unroll
                for (int c = 8 * h; c < 8 * h + 8; ++c) {  // this thread's 64 features
                    const uint32_t off = (c >> 3) * 16384 + (((c & 7) ^ (r & 7)) << 4);
                    cp_async_16_zfill(dq_s + off, srcq + c * 8, valid);
                    cp_async_16_zfill(dg_s + off, srcg + c * 8, valid);
                }
                if (h == 0) {
                    sL[r] = valid ? p.lse[lrow] * 1.4426950408889634f : INFINITY;
                    sD[r] = valid ? p.Dvec[lrow] : 0.f;
                    sRow[r] = valid ? qrow : -1;
                }
                cp_async_wait_all();
                fence_proxy_async_smem();
            }
            tc_fence_before();
            __syncthreads();
            tc_fence_after();
            // ---- S^T = K Q^T, dP^T = V dO^T
            if (threadIdx.x == 0) {
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t off = ((k >> 2) * 16384 + (k & 3) * 32) >> 4;
                    tc_mma_ss(tS, dK_k + off, dQ_k + off, idesc_ss, k > 0 ? 1u : 0u);
                }
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t off = ((k >> 2) * 16384 + (k & 3) * 32) >> 4;
                    tc_mma_ss(tP, dV_k + off, dG_k + off, idesc_ss, k > 0 ? 1u : 0u);
                }
                tc_commit(&bars->mma);
            }
            ok = tc_wait(&bars->mma, mma_phase & 1, abort_flag);
            if (!ok) BWD_NOTE(2, item, qt, mma_phase);
            if (!(ok = __syncthreads_and(ok))) break;
            ++mma_phase;
            tc_fence_after();
            // ---- P^T and dS^T for key r, 32 query columns at a time: this thread's two chunks
            // qq = 2h, 2h + 1 (queries 64h .. 64h + 63)
            {
                const int64_t key = u0 + r;
                const bool key_ok = r < ku;
#pragma unroll 1
                for (int qq = 2 * h; qq < 2 * h + 2; ++qq) {
                    uint32_t s32[32], g32[32];
                    tmem_ld32(tS + lane_off + qq * 32, s32);
                    tmem_ld32(tP + lane_off + qq * 32, g32);
                    tc_wait_ld();
                    uint32_t pk[16], dk2[16];
#pragma unroll
                    for (int i = 0; i < 32; i += 2) {
                        float pv[2], dsv[2];
#pragma unroll
                        for (int z = 0; z < 2; ++z) {
                            const int col = qq * 32 + i + z;  // query row of the tile
                            bool allowed = key_ok;
                            if (!past) allowed = allowed && key <= tdiag0 + col;
                            const float pe =
                                allowed ? ex2_approx(__uint_as_float(s32[i + z]) * p.scale_log2 - sL[col]) : 0.f;
                            pv[z] = pe;
                            dsv[z] = pe * (__uint_as_float(g32[i + z]) - sD[col]);
                        }
                        pk[i / 2] = pack_bf16x2(pv[0], pv[1]);
                        dk2[i / 2] = pack_bf16x2(dsv[0], dsv[1]);
                    }
                    // P^T over S columns [64h + 16 (qq - 2h), +16) and dS^T over the same dP columns:
                    // inside this thread's first chunk [64h, 64h + 32), which it has read, and which
                    // no other thread reads (queries 16k .. 16k + 15 end up at column 8k + 32 [k >= 4])
                    tmem_st16(tS + lane_off + 64 * h + 16 * (qq - 2 * h), pk);
                    tmem_st16(tP + lane_off + 64 * h + 16 * (qq - 2 * h), dk2);
                    // dS into shared memory, query-major: half qq / 2 holds queries 64 (qq / 2) .. +63,
                    // row r (this key) of 128 bytes, 16-byte chunks swizzled by (r & 7)
                    uint8_t* drow = sS + (qq >> 1) * 16384 + r * 128;
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4) {
                        const int c8 = (qq & 1) * 4 + c4;
                        const uint4 w = make_uint4(dk2[c4 * 4 + 0], dk2[c4 * 4 + 1], dk2[c4 * 4 + 2], dk2[c4 * 4 + 3]);
                        *reinterpret_cast<uint4*>(drow + ((c8 ^ (r & 7)) << 4)) = w;
                    }
                }
                tc_wait_st();
                fence_proxy_async_smem();
            }
            tc_fence_before();
            __syncthreads();
            tc_fence_after();
            // ---- dV += P^T dO, dK += dS^T Q, dQ = dS K (into S)
            if (threadIdx.x == 0) {
                const uint32_t first = qt == 0 ? 0u : 1u;  // the item's first tile starts dK, dV
                // packed P^T / dS^T of queries 16k .. 16k + 15 sit at column 8k (k < 4), 8k + 32 (k >= 4)
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    tc_mma_ts(tV, tS + k * 8 + (k >= 4 ? 32 : 0), dG_mn + k * 128, idesc_ts, (k > 0 || first) ? 1u : 0u);
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    tc_mma_ts(tK, tP + k * 8 + (k >= 4 ? 32 : 0), dQ_mn + k * 128, idesc_ts, (k > 0 || first) ? 1u : 0u);
#pragma unroll
                for (int k = 0; k < 8; ++k) tc_mma_ss(tS, dS_mn + k * 128, dK_mn + k * 128, idesc_dq, k > 0 ? 1u : 0u);
                tc_commit(&bars->mma);
            }
            ok = tc_wait(&bars->mma, mma_phase & 1, abort_flag);
            if (!ok) BWD_NOTE(3, item, qt, mma_phase);
            if (!(ok = __syncthreads_and(ok))) break;
            ++mma_phase;
            tc_fence_after();
            // ---- dQ row r (this query) into the accumulator: staged over the Q / dO / dS tiles (no
            // product reads them any more), then one bulk reduction per row
            {
                const int64_t dst = sRow[r];
                float* stage = (float*)(sQ + r * BWD_DQ_STRIDE);
#pragma unroll 1
                for (int c = 2 * h; c < 2 * h + 2; ++c) {  // this thread's half of the row
                    uint32_t v[32];
                    tmem_ld32(tS + lane_off + c * 32, v);
                    tc_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; i += 4)
                        *reinterpret_cast<uint4*>(stage + c * 32 + i) = make_uint4(v[i], v[i + 1], v[i + 2], v[i + 3]);
                }
                if (dst >= 0) {
                    fence_proxy_async_smem();  // the staged row is visible to the bulk-copy unit
                    bulk_reduce_add_f32(p.dq_acc + dst * MOBA_D + 64 * h, smem_u32(stage + 64 * h), MOBA_D * 2);
                    bulk_commit();
                }
                bulk_wait_read();  // the row is read before the next tile's gather overwrites it
            }
            tc_fence_before();
            __syncthreads();  // S, the tiles and the row tables are reused by the next tile
            tc_fence_after();
        }
        if (!ok) break;
        // ---- dK, dV of key r. tcgen05.ld is warp-collective (.sync.aligned): every lane loads, and
        // only the lanes of keys inside the step store (a partial last step has fewer keys).
        if (n_tiles > 0) {
            const bool key_ok = r < ku;
            const int64_t krow = ((int64_t)b * p.N + u0 + r) * p.Hkv + hk;
#pragma unroll 1
            for (int c = 2 * h; c < 2 * h + 2; ++c) {  // this thread's half of the features
                uint32_t a[32], v[32];
                tmem_ld32(tK + lane_off + c * 32, a);
                tmem_ld32(tV + lane_off + c * 32, v);
                tc_wait_ld();
                if (!key_ok) continue;
#pragma unroll
                for (int i = 0; i < 32; i += 8) {
                    uint4 wk, wv;
                    wk.x = pack_bf16x2(__uint_as_float(a[i]) * p.scale, __uint_as_float(a[i + 1]) * p.scale);
                    wk.y = pack_bf16x2(__uint_as_float(a[i + 2]) * p.scale, __uint_as_float(a[i + 3]) * p.scale);
                    wk.z = pack_bf16x2(__uint_as_float(a[i + 4]) * p.scale, __uint_as_float(a[i + 5]) * p.scale);
                    wk.w = pack_bf16x2(__uint_as_float(a[i + 6]) * p.scale, __uint_as_float(a[i + 7]) * p.scale);
                    wv.x = pack_bf16x2(__uint_as_float(v[i]), __uint_as_float(v[i + 1]));
                    wv.y = pack_bf16x2(__uint_as_float(v[i + 2]), __uint_as_float(v[i + 3]));
                    wv.z = pack_bf16x2(__uint_as_float(v[i + 4]), __uint_as_float(v[i + 5]));
                    wv.w = pack_bf16x2(__uint_as_float(v[i + 6]), __uint_as_float(v[i + 7]));
                    *reinterpret_cast<uint4*>(p.dk + krow * MOBA_D + c * 32 + i) = wk;
                    *reinterpret_cast<uint4*>(p.dv + krow * MOBA_D + c * 32 + i) = wv;
                }
            }
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    bulk_wait_all();  // this thread's dQ reductions are complete (and no longer read shared memory)
    // a wait that gave up may leave MMAs or loads in flight: give them a bounded time to land
    // before the shared memory and TMEM are released
    if (!ok && threadIdx.x == 0) {
        tc_commit(&bars->mma);
        int tmp = 0;
        tc_wait(&bars->mma, mma_phase & 1, &tmp, true, 200000000ull);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 512);
}
