// k_attn_tc.cuh - block-sparse attention on the sm_100a tensor cores.
//
// A work item is a pair of 128-row query tiles A and B that read the same keys
// (see k_attn_common.cuh), attended in steps of 128 keys ("MoBA project hub",
// Step 3; "NSA vs MoBA" blog, section 1 formula). For each tile X:
//   S_X = Q_X K^T                  tcgen05.mma, A = Q_X (smem), B = K (smem), D in TMEM
//   P_X = exp2(S_X * log2(e)/sqrt(d) - m_X)   softmax warps of X, one thread per TMEM lane
//   O_X += P_X V                   tcgen05.mma, A = P_X (TMEM, over S_X), B = V (smem)
// with a running row maximum m and sum l; the result is O / l and
// lse = (m + log2 l) * ln 2.
//
// Why pairs: one tile's steps form a strict chain (Q K^T -> softmax -> P V ->
// next Q K^T into the same S). Two tiles interleave on the tensor core - while
// the softmax warps of A work on S_A, the MMAs of B run - and each K/V step in
// shared memory feeds twice the MMA work.
//
// Roles (352 threads, one CTA per SM, persistent over the pairs):
//   warp 0     producer: lane 0 issues the TMA loads of K steps into a 3-slot ring
//              and of V steps into a 2-slot ring (3-D maps, 128-byte swizzle; K runs
//              one step ahead); the whole warp gathers each tile's Q rows (cp.async,
//              swizzled) as soon as the previous tile of the same X has issued its
//              last Q K^T, so a tile's rows arrive while the previous one finishes
//   warp 1     MMA issuer of tile A (and TMEM owner), warp 10 MMA issuer of tile B.
//              Per step i of a pair each issues [P V for step i-1, Q K^T for step i]
//              of its tile; the two alternate whole iterations through turn barriers
//              so the pipe runs one tile's batch, then the other's.
//   warps 2-5  softmax of tile A; warps 6-9 softmax of tile B. Each thread owns one
//              row: it runs the softmax with a lazily moved maximum and writes the
//              normalised row in the epilogue.
// Every role decodes an item from its 16-byte descriptor; the producer and the
// issuers load it an item ahead.
// TMEM: S_A [0,128), S_B [128,256), O_A [256,384), O_B [384,512) (fp32, 128 lanes).
// P_X (bf16 pairs) overwrites columns [64,128) of S_X once they have been read.
// The running maximum used for P only moves when the row maximum grows by more
// than 2^8 (log2 units), so O is rescaled rarely; P <= 2^8 stays exact in range.
//
// Ordering facts the waits rely on:
//   - the commit after Q K^T of X for step i also covers the P V of X for step
//     i - 1 issued before it, so "S_X ready" implies O_X holds every step so far;
//   - a parity wait for completion #k of a barrier is only sound when completion
//     #k-1 is known to have happened; each wait below says why it holds.
//
// Every wait is bounded. A wait that reaches its limit records
// MOBA_ERR_DEVICE_TIMEOUT and raises a CTA-wide abort flag; all roles then leave
// their loops, each MMA issuer waits (bounded) for its last MMAs, the producer
// for its loads in flight, and the TMEM is freed before the CTA exits.
#pragma once
#include <cuda.h>

#include "k_attn_common.cuh"

#define TC_THREADS 352
#define TC_KSLOTS 3
#define TC_VSLOTS 2
#define TC_STEP_BYTES 32768  // one K or V step: 128 keys x 128 d x bf16
#define TC_Q_BYTES 32768
#define TC_SMEM_BYTES (2 * TC_Q_BYTES + (TC_KSLOTS + TC_VSLOTS) * TC_STEP_BYTES + 512)
#define TC_RESCALE_LOG2 8.0f

struct __align__(64) TcMaps {
    CUtensorMap k;  // 3-D view (d, Hkv, B*N) of K, box (64, 1, 128), 128-byte swizzle
    CUtensorMap v;  // same for V
};

struct TcBars {
    uint64_t k_full[TC_KSLOTS], k_empty[TC_KSLOTS];
    uint64_t v_full[TC_VSLOTS], v_empty[TC_VSLOTS];
    uint64_t q_full[2];   // per tile: the producer warp's 32 lanes gathered its Q rows
    uint64_t q_empty[2];  // per tile: its last Q K^T has completed (Q_X may be refilled)
    uint64_t s_full[2];   // per tile: Q K^T of a step is in S_X (and P V of the previous step in O_X)
    uint64_t p_full[2];   // per tile: P_X of a step is in TMEM
    uint64_t o_full[2];   // per tile: the tile's last P V is in O_X
    uint64_t o_empty[2];  // per tile: the epilogue has read O_X
    uint64_t final_mma[2];  // per issuer: all of its MMAs have completed
    uint64_t turn[2];       // issuer x may issue its MMAs of the current iteration
    uint32_t tmem_base;
    int abort_flag;
    uint32_t k_issued[TC_KSLOTS], v_issued[TC_VSLOTS];  // loads issued per slot (teardown bookkeeping)
};

static_assert(sizeof(TcBars) <= 512, "barrier block does not fit the shared-memory budget");
static_assert(TC_SMEM_BYTES <= 227 * 1024, "over the per-block shared-memory limit");

__device__ __forceinline__ float max3f(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

__device__ __forceinline__ float row_max32(const uint32_t (&v)[32]) {
    float a0 = max3f(__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2]));
    float a1 = max3f(__uint_as_float(v[3]), __uint_as_float(v[4]), __uint_as_float(v[5]));
#pragma unroll
    for (int j = 6; j + 3 < 32; j += 4) {
        a0 = max3f(a0, __uint_as_float(v[j]), __uint_as_float(v[j + 1]));
        a1 = max3f(a1, __uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
    }
    return max3f(a0, a1, fmaxf(__uint_as_float(v[30]), __uint_as_float(v[31])));
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
#define EXP2_POLY_PAIRS 2  // of every 8 pairs of a step, evaluated by exp2_poly2 (2 measured best of 1-4)

// Masks the columns of a 64-key half (first column index c0) beyond `lim`.
__device__ __forceinline__ void mask_cols(uint32_t (&sr)[2][32], int c0, int lim) {
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int j = 0; j < 32; ++j)
            if (c0 + c * 32 + j > lim) sr[c][j] = __float_as_uint(-INFINITY);
}

// P = exp2(s * scale - m) for 64 keys into 32 bf16 pairs; returns their fp32 sum. The
// exponentials are split between the MUFU (ex2.approx) and the FMA pipe (exp2_poly2). A masked
// key (s = -inf) gets weight 0 on the MUFU path and 2^-126 on the FMA path (the clamp): next to
// the row maximum's weight >= 1 that is far below fp32 resolution in l and in O.
__device__ __forceinline__ float softmax_half(const uint32_t (&sr)[2][32], uint32_t (&pk)[32], float scale,
                                              float nm) {
    const uint64_t sc2 = f2pack(scale, scale), nm2 = f2pack(nm, nm);
    uint64_t acc2[2] = {0ull, 0ull};
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
            const uint64_t x2 = ffma2(f2pack(__uint_as_float(sr[c][j]), __uint_as_float(sr[c][j + 1])), sc2, nm2);
            uint64_t p2;
            if (((j >> 1) & 7) < EXP2_POLY_PAIRS) {
                p2 = exp2_poly2(x2);
            } else {
                float x0, x1;
                f2unpack(x2, x0, x1);
                p2 = f2pack(ex2_approx(x0), ex2_approx(x1));
            }
            acc2[(j >> 1) & 1] = fadd2(acc2[(j >> 1) & 1], p2);
            float p0, p1;
            f2unpack(p2, p0, p1);
            pk[c * 16 + (j >> 1)] = pack_bf16x2(p0, p1);
        }
    float l0, l1;
    f2unpack(fadd2(acc2[0], acc2[1]), l0, l1);
    return l0 + l1;
}

// Bounded wait that also gives up when another role raised the abort flag.
// `backoff` adds a short sleep between polls (for roles off the critical path,
// so their spinning does not take issue slots from the softmax warps).
// The limit is wall-clock time (limit_ns, MOBA_WAIT_NS by default), read every 256 polls.
__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                        bool backoff = false, uint64_t limit_ns = MOBA_WAIT_NS) {
    uint32_t n = 0;
    uint64_t t0 = 0;
    while (!mbar_try_wait(bar, parity)) {
        if (*abort_flag) return false;
        if ((++n & 255) == 0) {
            const uint64_t now = global_ns();
            if (t0 == 0) {
                t0 = now;
            } else if (now - t0 > limit_ns) {
                moba_set_error(MOBA_ERR_DEVICE_TIMEOUT);
                *abort_flag = 1;
                return false;
            }
        }
        if (backoff) __nanosleep(128);
    }
    return true;
}

// Failure-detection self-test: one warp waits, through tc_wait, on an mbarrier that
// nothing ever completes. The wait must give up after limit_ns, record
// MOBA_ERR_DEVICE_TIMEOUT and let the kernel return (no trap, no hang).
__global__ void __launch_bounds__(32) moba_wait_selftest_kernel(uint64_t limit_ns) {
    __shared__ uint64_t never;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&never, 1);
        abort_flag = 0;
        fence_mbarrier_init();
    }
    __syncwarp();
    tc_wait(&never, 0, &abort_flag, false, limit_ns);
}

// Warp-uniform form for roles whose next instruction is a .sync.aligned tcgen05 op.
__device__ __forceinline__ bool tc_wait_warp(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    const bool ok = tc_wait(bar, parity, abort_flag);
    return __all_sync(0xffffffffu, ok);
}


// Identity of row r of a tile: its query token and head, and for a past tile the slot of
// the partial (from the row's entry word en).
struct QRow {
    int64_t t;
    int hq, slot;
    bool valid;
};

__device__ __forceinline__ QRow q_row(const TileInfo& ti, uint64_t en, int r) {
    QRow q;
    if (ti.kind == 0) {
        q.valid = r < ti.ne;
        q.t = q.valid ? entry_t(en) : 0;
        q.hq = q.valid ? entry_hq(en) : 0;
        q.slot = q.valid ? entry_slot(en) : 0;
    } else {
        q.valid = r < ti.nt;
        q.t = ti.t0 + r;
        q.hq = ti.hq;
        q.slot = 0;
    }
    return q;
}

// Requests row r of a tile's Q into the swizzled tile (q_dst: the row's 128-byte line; 16-byte
// chunks XOR-swizzled by r & 7, the two 64-feature halves 16 KB apart). Rows past the tile's
// end are zero-filled. The caller waits for the copies.
__device__ __forceinline__ void gather_q_row(const AttnParams& a, const TileInfo& ti, const QRow& qr,
                                             uint32_t q_dst, int r) {
    const uint16_t* src = a.q + (qr.valid ? (((int64_t)ti.b * a.N + qr.t) * a.Hq + qr.hq) * MOBA_D : 0);
#pragma unroll
    for (int c = 0; c < 16; ++c)
        cp_async_16_zfill(q_dst + (c >> 3) * 16384 + (((c & 7) ^ (r & 7)) << 4), src + c * 8, qr.valid);
}

__global__ void __launch_bounds__(TC_THREADS, 1)
    moba_attn_tc_kernel(const AttnParams a, const __grid_constant__ TcMaps maps, int64_t items) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    if (smem_u32(smem_raw) & 1023) {  // the swizzled layout below needs a 1024-byte aligned window
        if (threadIdx.x == 0) moba_set_error(MOBA_ERR_UNSUPPORTED);
        return;
    }
    uint8_t* sQ = smem_raw;                                  // Q_A, Q_B: 2 x 32 KB
    uint8_t* sK = smem_raw + 2 * TC_Q_BYTES;                 // K ring
    uint8_t* sV = sK + TC_KSLOTS * TC_STEP_BYTES;            // V ring
    TcBars* bars = (TcBars*)(sV + TC_VSLOTS * TC_STEP_BYTES);
    volatile int* abort_flag = &bars->abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < TC_KSLOTS; ++s) {
            mbar_init(&bars->k_full[s], 1);
            mbar_init(&bars->k_empty[s], 2);  // one arrival per MMA issuer
            bars->k_issued[s] = 0;
        }
        for (int s = 0; s < TC_VSLOTS; ++s) {
            mbar_init(&bars->v_full[s], 1);
            mbar_init(&bars->v_empty[s], 2);
            bars->v_issued[s] = 0;
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(&bars->q_full[x], 32);
            mbar_init(&bars->q_empty[x], 1);
            mbar_init(&bars->s_full[x], 1);
            mbar_init(&bars->p_full[x], 128);
            mbar_init(&bars->o_full[x], 1);
            mbar_init(&bars->o_empty[x], 128);
        }
        mbar_init(&bars->final_mma[0], 1);
        mbar_init(&bars->final_mma[1], 1);
        mbar_init(&bars->turn[0], 1);
        mbar_init(&bars->turn[1], 1);
        bars->abort_flag = 0;
        fence_mbarrier_init();
        mbar_arrive(&bars->turn[0]);  // tile A's issuer goes first
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
        // ------------------------------------------------------------ producer warp
        // Lane 0 streams K and V. All 32 lanes gather Q: lane l takes rows l, l + 32, l + 64 and
        // l + 96 of a tile. An item's tiles are gathered after its first K step is requested and
        // before its first V step: the tile's first Q K^T needs Q and K0, its first P V comes
        // after a softmax. The entry words of the item's rows are loaded when the item starts.
        uint32_t gk = 0, gv = 0;  // K and V steps issued (lane 0)
        uint32_t nq[2] = {0, 0};  // tiles of A and of B gathered so far
        bool ok = true;
        auto load = [&](bool is_v, int hk, int row) -> bool {  // lane 0 only
            const uint32_t g = is_v ? gv : gk;
            const uint32_t nslots = is_v ? TC_VSLOTS : TC_KSLOTS;
            const uint32_t s = g % nslots;
            uint64_t* full = is_v ? &bars->v_full[s] : &bars->k_full[s];
            uint64_t* empty = is_v ? &bars->v_empty[s] : &bars->k_empty[s];
            // completion #(g/n - 1) of the slot's empty barrier; #(g/n - 2) was waited n loads ago
            if (!tc_wait(empty, ((g / nslots) & 1) ^ 1, abort_flag, true)) return false;
            uint8_t* dst = (is_v ? sV : sK) + s * TC_STEP_BYTES;
            const void* map = is_v ? (const void*)&maps.v : (const void*)&maps.k;
            mbar_arrive_expect_tx(full, TC_STEP_BYTES);
            tma_load_3d(smem_u32(dst), map, full, 0, hk, row);
            tma_load_3d(smem_u32(dst + 16384), map, full, 64, hk, row);
            if (is_v) {
                bars->v_issued[s] += 1;
                ++gv;
            } else {
                bars->k_issued[s] += 1;
                ++gk;
            }
            return true;
        };
        PairDesc dn = pair_desc(a, blockIdx.x);
        for (int64_t item = blockIdx.x; item < items && ok; item += gridDim.x) {
            const PairDesc d = dn;
            if (item + gridDim.x < items) dn = pair_desc(a, item + gridDim.x);  // an item ahead
            const PairInfo pi = decode_pair(a, item, d);
            if (pi.ns == 0) continue;
            uint64_t ew[2][4];  // entry words of this lane's rows (past tiles)
#pragma unroll
            for (int x = 0; x < 2; ++x)
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int rr = lane + 32 * k;
                    ew[x][k] = (pi.t[x].kind == 0 && rr < pi.t[x].ne) ? a.entries[pi.t[x].e0 + rr] : 0ull;
                }
            const bool first = pi.t[0].kind >= 0;
            const int hk = first ? pi.t[0].hk : pi.t[1].hk;
            const int64_t row0 = (int64_t)(first ? pi.t[0].b : pi.t[1].b) * a.N + (first ? pi.t[0].klo : pi.t[1].klo);
            if (lane == 0) ok = load(false, hk, (int)row0);  // K0
            if (!(ok = __shfl_sync(0xffffffffu, ok, 0))) break;
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                const TileInfo& ti = pi.t[x];
                if (ti.kind < 0) continue;
                // completion #nq-1 of q_empty[x]: the previous tile of x has read Q_x for the last
                // time (for the first tile the wait returns at once); #nq-2 was waited before the
                // previous gather
                if (!(ok = tc_wait_warp(&bars->q_empty[x], (nq[x] & 1) ^ 1, abort_flag))) break;
                const uint32_t base = smem_u32(sQ + x * TC_Q_BYTES);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int rr = lane + 32 * k;
                    gather_q_row(a, ti, q_row(ti, ew[x][k], rr), base + rr * 128, rr);
                }
                cp_async_wait_all();
                fence_proxy_async_smem();
                mbar_arrive(&bars->q_full[x]);
                ++nq[x];
            }
            if (!ok) break;
            if (lane == 0) {  // K one step ahead of V: K0, K1, V0, K2, V1, ...
                for (int64_t i = 0; i < pi.ns; ++i) {
                    if (i + 1 < pi.ns && !(ok = load(false, hk, (int)(row0 + (i + 1) * MOBA_KCHUNK)))) break;
                    if (!(ok = load(true, hk, (int)(row0 + i * MOBA_KCHUNK)))) break;
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
        }
        cp_async_wait_all();  // no copy may still write the shared memory when the CTA leaves
        __syncwarp();
    } else if (warp == 1 || warp == TC_THREADS / 32 - 1) {
        // ------------------------------------------------------------ MMA issuers
        // One warp per tile (warp 1: tile A, the last warp: tile B), so each tile's P V and
        // Q K^T go out as soon as its own P is ready, and one issuer's waits do not hold back
        // the other's MMAs. Both walk the same pairs and K/V steps and release every K/V slot
        // once (count 2 on the empty barriers): with a commit after using it, or with a plain
        // arrive when their tile has no work in that step. The warp runs converged, so every
        // descriptor and counter is warp-uniform; the elected lane (lane 0 of the full warp,
        // always the same thread) issues each MMA and commit, so a commit covers all of them.
        const int x = warp == 1 ? 0 : 1;
        const uint32_t tS = tmem + x * 128, tO = tmem + 256 + x * 128;
        const uint32_t idesc_qk = make_idesc_bf16(128, 128, 0, 0);
        const uint32_t idesc_pv = make_idesc_bf16(128, 128, 0, 1);
        // descriptors of this tile's Q buffer and of the first K and V buffers; the other slots
        // follow at fixed offsets (the start-address field is addr >> 4; all buffers end below 256 KB)
        const uint64_t dq = make_sdesc_sw128(smem_u32(sQ + x * TC_Q_BYTES), 16, 1024);
        const uint64_t dk0 = make_sdesc_sw128(smem_u32(sK), 16, 1024);
        const uint64_t dv0 = make_sdesc_sw128(smem_u32(sV), 16384, 1024);
        uint32_t gk = 0, gv = 0;  // K / V steps consumed
        uint32_t px = 0, tx = 0;  // P V steps issued, tiles finished
        uint32_t it = 0;          // iterations of the issue loop (the same sequence for both issuers)
        bool ok = true;
        PairDesc dn = pair_desc(a, blockIdx.x);
        for (int64_t item = blockIdx.x; item < items && ok; item += gridDim.x) {
            const PairDesc d = dn;
            if (item + gridDim.x < items) dn = pair_desc(a, item + gridDim.x);  // an item ahead
            const PairInfo pi = decode_pair(a, item, d);
            if (pi.ns == 0) continue;
            const int64_t nx = tile_steps(x ? pi.t[1] : pi.t[0]);
            // completion #tx of q_full[x]: #tx-1 was waited for the previous tile of x
            if (nx > 0 && !(ok = tc_wait_warp(&bars->q_full[x], tx & 1, abort_flag))) break;
            for (int64_t i = 0; i <= pi.ns && ok; ++i) {
                const bool do_qk = i < pi.ns, do_pv = i > 0;
                const bool my_qk = do_qk && i < nx, my_pv = do_pv && i - 1 < nx;
                const uint32_t ks = gk % TC_KSLOTS, vs = gv % TC_VSLOTS;
                // The K/V waits come first (those loads were issued long ago, P is the real gate).
                // An issuer waits for every step's K and V even when its tile has no work in that
                // step: its release of the slot below must not come before the slot was filled, or
                // it would count toward the slot's previous use (completion #g/n - 1 of the empty
                // barrier, which the producer waited for before this load).
                if (do_pv && !(ok = tc_wait_warp(&bars->v_full[vs], (gv / TC_VSLOTS) & 1, abort_flag))) break;
                if (do_qk && !(ok = tc_wait_warp(&bars->k_full[ks], (gk / TC_KSLOTS) & 1, abort_flag))) break;
                // O_x is free once the previous tile's epilogue has read it
                if (my_pv && i == 1 && !(ok = tc_wait_warp(&bars->o_empty[x], (tx & 1) ^ 1, abort_flag))) break;
                // Turns: the issuers alternate whole iterations (A, B, A, ...), so the tensor pipe
                // runs one tile's batch before the other's and the two softmax groups stay out of
                // phase (each softmax runs while the other tile's MMAs do). Completion #it of
                // turn[x] is the other issuer's hand-over after its iteration it - 1 (for tile A's
                // first iteration the initial arrival); #it-1 was waited at the previous iteration.
                if (!(ok = tc_wait_warp(&bars->turn[x], it & 1, abort_flag))) break;
                // P last: in steady state it is the event that gates the iteration.
                // Completion #px of p_full[x]; #px-1 was waited before the previous P V.
                if (my_pv && !(ok = tc_wait_warp(&bars->p_full[x], px & 1, abort_flag))) break;
                tc_fence_after();
                if (my_pv) {
                    const uint64_t vd = dv0 + (uint64_t)(vs * (TC_STEP_BYTES >> 4));
                    tc_mma_ts_w(tO, tS + 64, vd, idesc_pv, i > 1 ? 1u : 0u);
#pragma unroll
                    for (int k = 1; k < 8; ++k) tc_mma_ts_w(tO, tS + 64 + k * 8, vd + k * 128, idesc_pv, 1u);
                    ++px;
                    if (i == nx) {  // that was the tile's last step
                        tc_commit_w(&bars->o_full[x]);
                        ++tx;
                    }
                }
                if (my_qk) {
                    const uint64_t kd = dk0 + (uint64_t)(ks * (TC_STEP_BYTES >> 4));
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const uint32_t off = ((k >> 2) * 16384 + (k & 3) * 32) >> 4;
                        tc_mma_ss_w(tS, dq + off, kd + off, idesc_qk, k > 0 ? 1u : 0u);
                    }
                    tc_commit_w(&bars->s_full[x]);
                    if (i + 1 == nx) tc_commit_w(&bars->q_empty[x]);  // the tile's last read of Q_x
                }
                mbar_arrive_w(&bars->turn[x ^ 1]);
                ++it;
                if (do_qk) {  // this issuer is done with K step gk
                    if (my_qk) tc_commit_w(&bars->k_empty[ks]);
                    else mbar_arrive_w(&bars->k_empty[ks]);
                    ++gk;
                }
                if (do_pv) {  // and with V step gv
                    if (my_pv) tc_commit_w(&bars->v_empty[vs]);
                    else mbar_arrive_w(&bars->v_empty[vs]);
                    ++gv;
                }
            }
        }
        // all MMAs of this issuer have completed before TMEM is released
        __syncwarp();
        tc_commit_w(&bars->final_mma[x]);
        mbar_wait(&bars->final_mma[x], 0);
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax warps
        const int x = (warp - 2) >> 2;           // tile of the pair handled by this warp group
        const int r = 32 * (warp & 3) + lane;    // tile row == TMEM lane
        const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
        const uint32_t tS = tmem + x * 128 + lane_off;
        const uint32_t tO = tmem + 256 + x * 128 + lane_off;
        uint32_t g = 0, tile_i = 0;
        for (int64_t item = blockIdx.x; item < items; item += gridDim.x) {
            const PairInfo pi = decode_pair(a, item);
            const TileInfo ti = x ? pi.t[1] : pi.t[0];  // by value: stays in registers
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
            // last key column this row may read, relative to the tile's first key: the key range
            // and, on the own block, causality (u <= t)
            int lim0;
            {
                int64_t last = ti.khi - 1;
                if (ti.kind != 0 && t < last) last = t;
                lim0 = (int)(last - ti.klo);
            }
            // output row: the slot's partial for a past tile, out / lse for an own-block tile
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
            float m_used = -INFINITY, l = 0.f;
            bool ok = true;
            for (uint32_t i = 0; i < nst; ++i) {
                const uint32_t gg = g + i;
                // completion #gg of s_full[x]; #gg-1 was waited at the previous step
                if (!(ok = tc_wait_warp(&bars->s_full[x], gg & 1, abort_flag))) break;
                tc_fence_after();
                const int lim = lim0 - (int)i * MOBA_KCHUNK;  // last allowed column of this step
                const bool full = lim >= MOBA_KCHUNK - 1;
                if (i == 0) {
                    // The running maximum starts at the first step's row maximum (finite: column 0
                    // of a tile's first step is allowed for every row), so that step never rescales.
                    uint32_t sm[2][32];
                    tmem_ld32(tS, sm[0]);
                    tmem_ld32(tS + 32, sm[1]);
                    tc_wait_ld();
                    if (!full) mask_cols(sm, 0, lim);
                    float mx = fmaxf(row_max32(sm[0]), row_max32(sm[1]));
                    tmem_ld32(tS + 64, sm[0]);
                    tmem_ld32(tS + 96, sm[1]);
                    tc_wait_ld();
                    if (!full) mask_cols(sm, 64, lim);
                    mx = fmaxf(mx, fmaxf(row_max32(sm[0]), row_max32(sm[1])));
                    m_used = mx * a.scale_log2;
                }
                // P against the running maximum. S columns [0,64) are read and their P computed,
                // then columns [64,128) are read into registers, and only then is the first P
                // stored over columns [64,96) (already read). If the step's maximum moved the
                // running one by more than the threshold, the overwritten S columns are put back
                // from registers, O and l are rescaled and the step is done again (rare: the
                // first step already fixed the scale).
                for (;;) {
                    const float nm = -m_used;
                    uint32_t s1[2][32];
                    float mx, lsum;
                    {
                        uint32_t pk0[32];
                        {
                            uint32_t s0[2][32];
                            tmem_ld32(tS, s0[0]);
                            tmem_ld32(tS + 32, s0[1]);
                            tc_wait_ld();
                            if (!full) mask_cols(s0, 0, lim);
                            mx = fmaxf(row_max32(s0[0]), row_max32(s0[1]));
                            lsum = softmax_half(s0, pk0, a.scale_log2, nm);
                        }
                        tmem_ld32(tS + 64, s1[0]);
                        tmem_ld32(tS + 96, s1[1]);
                        tc_wait_ld();
                        tmem_st32(tS + 64, pk0);
                    }
                    if (!full) mask_cols(s1, 64, lim);
                    mx = fmaxf(mx, fmaxf(row_max32(s1[0]), row_max32(s1[1])));
                    const float m_new = fmaxf(m_used, mx * a.scale_log2);
                    if (__any_sync(0xffffffffu, m_new > m_used + TC_RESCALE_LOG2)) {
                        tmem_st32(tS + 64, s1[0]);  // S columns [64,96) again (masked ones stay masked)
                        const float f = ex2_approx(m_used - m_new);
                        // O_x holds P V of every earlier step (S ready implies it); i > 0 here
#pragma unroll 1
                        for (int c = 0; c < 4; ++c) {
                            uint32_t o[32];
                            tmem_ld32(tO + c * 32, o);
                            tc_wait_ld();
#pragma unroll
                            for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * f);
                            tmem_st32(tO + c * 32, o);
                        }
                        l *= f;
                        m_used = m_new;
                        tc_wait_st();  // the restored S columns land before they are read again
                        continue;
                    }
                    uint32_t pk1[32];
                    lsum += softmax_half(s1, pk1, a.scale_log2, nm);
                    tmem_st32(tS + 96, pk1);
                    l += lsum;
                    break;
                }
                tc_wait_st();
                tc_fence_before();
                mbar_arrive(&bars->p_full[x]);
            }
            if (!ok) break;
            // epilogue: completion #tile_i of o_full[x]; #tile_i-1 was waited at the previous tile
            if (!tc_wait_warp(&bars->o_full[x], tile_i & 1, abort_flag)) break;
            tc_fence_after();
            const float inv = 1.f / l;
#pragma unroll 1
            for (int hh = 0; hh < 2; ++hh) {  // 64 output features at a time
                uint32_t ob[2][32];
                tmem_ld32(tO + hh * 64, ob[0]);
                tmem_ld32(tO + hh * 64 + 32, ob[1]);
                tc_wait_ld();
                if (hh == 1) {  // O_x has been read: the next tile may overwrite it
                    tc_fence_before();
                    mbar_arrive(&bars->o_empty[x]);
                }
                if (valid) {
#pragma unroll
                    for (int c = 0; c < 2; ++c)
#pragma unroll
                        for (int j = 0; j < 32; j += 8) {
                            uint4 w;
                            w.x = pack_bf16x2(__uint_as_float(ob[c][j + 0]) * inv, __uint_as_float(ob[c][j + 1]) * inv);
                            w.y = pack_bf16x2(__uint_as_float(ob[c][j + 2]) * inv, __uint_as_float(ob[c][j + 3]) * inv);
                            w.z = pack_bf16x2(__uint_as_float(ob[c][j + 4]) * inv, __uint_as_float(ob[c][j + 5]) * inv);
                            w.w = pack_bf16x2(__uint_as_float(ob[c][j + 6]) * inv, __uint_as_float(ob[c][j + 7]) * inv);
                            *reinterpret_cast<uint4*>(dst + hh * 64 + c * 32 + j) = w;
                        }
                }
            }
            if (valid) *ldst = (m_used + __log2f(l)) * 0.69314718055994530942f;
            g += nst;
            tile_i += 1;
        }
    }

    // ---------------------------------------------------------------- teardown
    __syncthreads();
    if (warp == 0 && lane == 0 && *abort_flag) {
        // let every load already issued land before the shared memory goes away
        for (int s = 0; s < TC_KSLOTS; ++s)
            if (bars->k_issued[s] > 0) mbar_wait(&bars->k_full[s], (bars->k_issued[s] - 1) & 1);
        for (int s = 0; s < TC_VSLOTS; ++s)
            if (bars->v_issued[s] > 0) mbar_wait(&bars->v_full[s], (bars->v_issued[s] - 1) & 1);
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
    {
        const cudaError_t err =
            cudaFuncSetAttribute(moba_attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, TC_SMEM_BYTES);
        if (err != cudaSuccess) {
            moba_note_cuda_error(err);
            return MOBA_ERR_CUDA;
        }
    }
    const int64_t grid = items < nsm ? items : nsm;  // one CTA per SM, striped over the pairs
    moba_attn_tc_kernel<<<(unsigned)grid, TC_THREADS, TC_SMEM_BYTES, st>>>(a, maps, items);
    const cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) {
        cudaGetLastError();
        (void)cudaPeekAtLastError();
        moba_note_cuda_error(err);
        return MOBA_ERR_CUDA;
    }
    return MOBA_OK;
}
