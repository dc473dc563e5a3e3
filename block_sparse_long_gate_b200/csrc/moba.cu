// moba.cu - the C ABI of libmoba: argument checks, workspace layout and the
// launch sequence of the MoBA causal prefill forward on one sm_100a GPU.
//
//   pool (K -> Kbar) -> gate (Q, Kbar -> idx) -> count / scan / scatter
//   (idx -> per-block query lists) -> attention tiles (past blocks -> partials,
//   own block -> out / lse) -> merge (partials -> out / lse)
//
// Everything after the host-side checks is queued on the caller's stream; no
// call synchronises the device.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "k_attn_common.cuh"
#include "k_attn_simt.cuh"
#include "k_attn_tc.cuh"
#include "k_backward.cuh"
#include "k_decode.cuh"
#include "k_gate.cuh"
#include "k_gate_tc.cuh"
#include "k_invert.cuh"
#include "k_merge.cuh"
#include "k_pool.cuh"

namespace {

// Test hooks (process-wide): 0 = the default kernels, 1 = the CUDA-core cross-check kernels.
std::atomic<int> g_attn_impl{0};  // attention: 0 tensor cores, 1 CUDA cores
std::atomic<int> g_gate_impl{0};  // gate: 0 tensor cores + exact boundary, 1 CUDA-core fp64

// Kernel launches made by the library (all devices, all threads).
std::atomic<uint64_t> g_launches{0};

// Optional per-stage timing: CUDA events recorded between the stages of each
// forward call, on the call's stream.
constexpr int kStages = 5;  // pool, gate, invert, attention, merge
struct StageRec {
    cudaEvent_t ev[kStages + 1];
};
std::mutex g_timing_mu;
bool g_timing = false;
std::vector<StageRec> g_recs;

struct StageTimer {
    StageRec rec;
    bool on = false;
    cudaStream_t st;
    explicit StageTimer(cudaStream_t s) : st(s) {
        std::lock_guard<std::mutex> lk(g_timing_mu);
        if (!g_timing) return;
        on = true;
        for (int i = 0; i <= kStages; ++i)
            if (cudaEventCreate(&rec.ev[i]) != cudaSuccess) on = false;
        if (on) cudaEventRecord(rec.ev[0], st);
    }
    void mark(int stage) {  // end of stage `stage` (0-based)
        if (on) cudaEventRecord(rec.ev[stage + 1], st);
    }
    void finish(int upto) {
        if (!on) return;
        for (int i = upto; i < kStages; ++i) cudaEventRecord(rec.ev[i + 1], st);
        std::lock_guard<std::mutex> lk(g_timing_mu);
        g_recs.push_back(rec);
    }
};

inline void count_launch(int n = 1) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

// Text of the last CUDA error the library saw on this host thread.
thread_local const char* g_last_cuda_error = "no error";

inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct Plan {
    int B, Hq, Hkv, G, d, bs, topk, kp;
    int64_t N, nblk, nfull, L, nch, E, Pmax, D, mb, ml, per_bh, nseg, nscan_parts;
    size_t off_kbar, off_planes, off_mu, off_stats, off_idx, off_counts, off_segoff, off_tiles, off_parts, off_entries,
        off_items, off_opart, off_lpart, gate_bytes;
    size_t total;
};

int make_plan(int B, int Hq, int Hkv, int64_t N, int d, int bs, int topk, Plan* p) {
    if (B < 1 || Hq < 1 || Hkv < 1 || N < 1 || bs < 1 || topk < 1) return MOBA_ERR_SHAPE;
    if (d != MOBA_D || Hq % Hkv != 0 || topk > MOBA_MAX_TOPK || N >= ((int64_t)1 << 31)) return MOBA_ERR_SHAPE;
    if (B > 65535 || Hq > 65535) return MOBA_ERR_SHAPE;
    if ((int64_t)B * N >= ((int64_t)1 << 31)) return MOBA_ERR_SHAPE;  // TMA row coordinates are 32-bit
    Plan& P = *p;
    P.B = B;
    P.Hq = Hq;
    P.Hkv = Hkv;
    P.G = Hq / Hkv;
    P.d = d;
    P.bs = bs;
    P.topk = topk;
    P.kp = topk - 1;
    P.N = N;
    P.nblk = cdiv(N, bs);
    if (P.nblk > MOBA_MAX_BLOCKS) return MOBA_ERR_SHAPE;  // per-block counters live in shared memory
    P.nfull = N / bs;
    P.L = (int64_t)B * Hkv * P.nblk;
    if (P.L >= ((int64_t)1 << 31)) return MOBA_ERR_SHAPE;  // a pair descriptor holds its list in 32 bits
    P.nch = cdiv(N, INV_CHUNK);
    // exact number of earlier-block selections of well-formed rows: sum_t min(c(t), k - 1)
    int64_t per_head = 0;
    for (int64_t c = 0; c < P.nblk; ++c) {
        int64_t n_c = (c * bs + bs <= N) ? bs : N - c * bs;
        per_head += n_c * (c < P.kp ? c : P.kp);
    }
    P.E = per_head * B * Hq;
    P.Pmax = P.E / MOBA_PAIR_ROWS + P.L;  // past pairs: <= 256 entries of one list each
    P.mb = cdiv(bs, MOBA_TILE);
    int64_t nlast = N - (P.nblk - 1) * bs;
    P.ml = cdiv(nlast, MOBA_TILE);
    P.per_bh = (P.nblk - 1) * cdiv(P.mb, 2) + cdiv(P.ml, 2);  // own-block pairs per (b, hq)
    P.D = (int64_t)B * Hq * P.per_bh;
    P.nseg = P.L * P.nch;
    int64_t nscan = P.nseg > P.L ? P.nseg : P.L;
    P.nscan_parts = cdiv(nscan, SCAN_TILE);

    size_t o = 0;
    const size_t nf = (size_t)(P.nfull > 0 ? P.nfull : 1);
    P.off_kbar = o;
    o = align256(o + sizeof(double) * (size_t)B * Hkv * nf * MOBA_D);
    P.off_planes = o;
    o = align256(o + sizeof(uint16_t) * (size_t)B * Hkv * 2 * nf * MOBA_D);
    P.off_mu = o;
    o = align256(o + sizeof(float) * (size_t)B * Hkv * nf);
    P.off_stats = o;
    o = align256(o + sizeof(unsigned) * (size_t)B * Hkv * 2);
    P.gate_bytes = o;  // the gate's scratch is the workspace's first gate_bytes bytes
    P.off_idx = o;
    o = align256(o + sizeof(int32_t) * (size_t)B * Hq * N * topk);
    P.off_counts = o;
    o = align256(o + sizeof(uint32_t) * (size_t)P.nseg);
    P.off_segoff = o;
    o = align256(o + sizeof(int64_t) * (size_t)(P.nseg + 1));
    P.off_tiles = o;
    o = align256(o + sizeof(int64_t) * (size_t)(P.L + 1));
    P.off_parts = o;
    o = align256(o + sizeof(int64_t) * (size_t)P.nscan_parts);
    P.off_entries = o;
    o = align256(o + sizeof(uint64_t) * (size_t)(P.E > 0 ? P.E : 1));
    P.off_items = o;
    o = align256(o + sizeof(PairDesc) * (size_t)(P.Pmax > 0 ? P.Pmax : 1));
    P.off_opart = o;
    o = align256(o + sizeof(uint16_t) * (size_t)B * Hq * N * (P.kp > 0 ? P.kp : 1) * MOBA_D);
    P.off_lpart = o;
    o = align256(o + sizeof(float) * (size_t)B * Hq * N * (P.kp > 0 ? P.kp : 1));
    P.total = o;
    return MOBA_OK;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15) == 0; }

// Records the text of a failed CUDA call for moba_last_error_string() and resets the
// runtime's last-error state.
int cuda_fail(cudaError_t e) {
    g_last_cuda_error = cudaGetErrorString(e);
    cudaGetLastError();
    return MOBA_ERR_CUDA;
}

int check_device() {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    int major = 0, minor = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess) return cuda_fail(e);
    if ((e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess) return cuda_fail(e);
    if (major != 10 || minor != 0) return MOBA_ERR_UNSUPPORTED;
    return MOBA_OK;
}

int check_ptrs(std::initializer_list<const void*> ps) {
    for (const void* p : ps)
        if (!p) return MOBA_ERR_NULL;
    for (const void* p : ps)
        if (!aligned16(p)) return MOBA_ERR_ALIGN;
    return MOBA_OK;
}

}  // namespace

void moba_note_cuda_error(cudaError_t e) { g_last_cuda_error = cudaGetErrorString(e); }

namespace {

int launch_ok() {
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? MOBA_OK : cuda_fail(e);
}

// ---------------------------------------------------------------- stages
// Gate scratch inside a workspace: Kbar (fp64) and, for the tensor-core gate, the centre /
// residual-plane form of it and the per-head magnitude bounds.
struct GateScratch {
    double* kbar;
    PoolAux aux;  // all null: fp64 gate only
};

GateScratch gate_scratch(const Plan& P, char* ws, bool tc) {
    GateScratch g;
    g.kbar = (double*)(ws + P.off_kbar);
    g.aux.planes = tc ? (uint16_t*)(ws + P.off_planes) : nullptr;
    g.aux.mu = tc ? (float*)(ws + P.off_mu) : nullptr;
    g.aux.head_stats = tc ? (unsigned*)(ws + P.off_stats) : nullptr;
    return g;
}

bool use_tc_gate(const Plan& P) { return g_gate_impl.load() == 0 && P.nfull > 0 && P.kp > 0; }

int run_pool(const Plan& P, const void* k, const GateScratch& gs, PoolMode pm, cudaStream_t st) {
    if (P.nfull == 0) return MOBA_OK;
    if (gs.aux.head_stats) {
        const cudaError_t e = cudaMemsetAsync(gs.aux.head_stats, 0, sizeof(unsigned) * 2 * (size_t)P.B * P.Hkv, st);
        if (e != cudaSuccess) return cuda_fail(e);
    }
    dim3 grid((unsigned)P.nfull, P.Hkv, P.B);
    moba_pool_kernel<<<grid, POOL_THREADS, 0, st>>>((const uint16_t*)k, gs.kbar, P.N, P.Hkv, P.bs, P.nfull,
                                                    gs.aux, pm);
    count_launch();
    return launch_ok();
}

int run_gate_simt(const Plan& P, const void* q, const double* kbar, int32_t* idx, cudaStream_t st);

int run_gate(const Plan& P, const void* q, const GateScratch& gs, int32_t* idx, cudaStream_t st) {
    if (!gs.aux.planes) return run_gate_simt(P, q, gs.kbar, idx, st);
    GateParams gp;
    gp.q = (const uint16_t*)q;
    gp.kbar = gs.kbar;
    gp.mu = gs.aux.mu;
    gp.stats = gs.aux.head_stats;
    gp.idx = idx;
    gp.N = P.N;
    gp.nfull = P.nfull;
    gp.tiles_per_head = cdiv(P.N, 128);
    gp.ntiles = gp.tiles_per_head * P.B * P.Hq;
    gp.B = P.B;
    gp.Hq = P.Hq;
    gp.Hkv = P.Hkv;
    gp.G = P.G;
    gp.bs = P.bs;
    gp.topk = P.topk;
    gp.kp = P.kp;
    const int rc = run_gate_tc(gp, gs.aux.planes, st);
    if (rc == MOBA_OK) count_launch();
    return rc;
}

int run_gate_simt(const Plan& P, const void* q, const double* kbar, int32_t* idx, cudaStream_t st) {
    dim3 grid((unsigned)cdiv(P.N, GATE_ROWS), P.Hq, P.B);
    const uint16_t* qq = (const uint16_t*)q;
    if (P.kp <= 8)
        moba_gate_simt_kernel<8><<<grid, GATE_ROWS, 0, st>>>(qq, kbar, idx, P.N, P.Hq, P.Hkv, P.bs, P.topk, P.nfull);
    else if (P.kp <= 16)
        moba_gate_simt_kernel<16><<<grid, GATE_ROWS, 0, st>>>(qq, kbar, idx, P.N, P.Hq, P.Hkv, P.bs, P.topk, P.nfull);
    else if (P.kp <= 32)
        moba_gate_simt_kernel<32><<<grid, GATE_ROWS, 0, st>>>(qq, kbar, idx, P.N, P.Hq, P.Hkv, P.bs, P.topk, P.nfull);
    else
        moba_gate_simt_kernel<64><<<grid, GATE_ROWS, 0, st>>>(qq, kbar, idx, P.N, P.Hq, P.Hkv, P.bs, P.topk, P.nfull);
    count_launch();
    return launch_ok();
}

int run_scan(ScanSrc src, int64_t n, int64_t* parts, int64_t* out, cudaStream_t st) {
    int64_t nb = cdiv(n, SCAN_TILE);
    moba_scan_partial_kernel<<<(unsigned)nb, SCAN_THREADS, 0, st>>>(src, n, parts);
    moba_scan_top_kernel<<<1, SCAN_THREADS, 0, st>>>(parts, nb);
    moba_scan_final_kernel<<<(unsigned)nb, SCAN_THREADS, 0, st>>>(src, n, parts, out);
    count_launch(3);
    return launch_ok();
}

int run_invert(const Plan& P, const int32_t* idx, char* ws, cudaStream_t st) {
    uint32_t* counts = (uint32_t*)(ws + P.off_counts);
    int64_t* segoff = (int64_t*)(ws + P.off_segoff);
    int64_t* tiles = (int64_t*)(ws + P.off_tiles);
    int64_t* parts = (int64_t*)(ws + P.off_parts);
    uint64_t* entries = (uint64_t*)(ws + P.off_entries);
    dim3 grid((unsigned)P.nch, P.Hkv, P.B);
    size_t sm_count = sizeof(uint32_t) * (size_t)P.nblk;
    size_t sm_scatter = (sizeof(int64_t) + sizeof(uint32_t)) * (size_t)P.nblk;
    cudaError_t e = cudaFuncSetAttribute(moba_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_count);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(moba_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_scatter);
    if (e != cudaSuccess) return cuda_fail(e);
    moba_count_kernel<<<grid, INV_THREADS, sm_count, st>>>(idx, counts, P.N, P.Hq, P.Hkv, P.bs, P.topk, P.nblk,
                                                           P.nch);
    count_launch();
    int rc = launch_ok();
    if (rc) return rc;
    ScanSrc s1{counts, nullptr, 0};
    if ((rc = run_scan(s1, P.nseg, parts, segoff, st))) return rc;
    ScanSrc s2{nullptr, segoff, P.nch};
    if ((rc = run_scan(s2, P.L, parts, tiles, st))) return rc;
    if (P.Pmax > 0) {
        moba_item_list_kernel<<<(unsigned)cdiv(P.Pmax, SCAN_THREADS), SCAN_THREADS, 0, st>>>(
            tiles, segoff, P.L, P.nch, P.Pmax, (PairDesc*)(ws + P.off_items));
        count_launch();
        if ((rc = launch_ok())) return rc;
    }
    moba_scatter_kernel<<<grid, INV_THREADS, sm_scatter, st>>>(idx, segoff, entries, P.N, P.Hq, P.Hkv, P.bs,
                                                               P.topk, P.nblk, P.nch);
    count_launch();
    return launch_ok();
}

AttnParams attn_params(const Plan& P, const void* q, const void* k, const void* v, void* out, float* lse,
                       char* ws) {
    AttnParams a;
    a.q = (const uint16_t*)q;
    a.k = (const uint16_t*)k;
    a.v = (const uint16_t*)v;
    a.N = P.N;
    a.B = P.B;
    a.Hq = P.Hq;
    a.Hkv = P.Hkv;
    a.G = P.G;
    a.bs = P.bs;
    a.topk = P.topk;
    a.kp = P.kp;
    a.nblk = P.nblk;
    a.nch = P.nch;
    a.entries = ws ? (const uint64_t*)(ws + P.off_entries) : nullptr;
    a.segoff = ws ? (const int64_t*)(ws + P.off_segoff) : nullptr;
    a.pairs = ws ? (const PairDesc*)(ws + P.off_items) : nullptr;
    a.L = P.L;
    a.Pmax = P.Pmax;
    a.opart = ws ? (uint16_t*)(ws + P.off_opart) : nullptr;
    a.lpart = ws ? (float*)(ws + P.off_lpart) : nullptr;
    a.D = P.D;
    a.mb = P.mb;
    a.ml = P.ml;
    a.per_bh = P.per_bh;
    a.dense = 0;
    a.out = (uint16_t*)out;
    a.lse = lse;
    a.scale_log2 = (float)(1.4426950408889634 / sqrt((double)P.d));
    return a;
}

int run_attention(const Plan& P, const AttnParams& a, cudaStream_t st) {
    const int64_t items = a.Pmax + a.D;
    if (g_attn_impl.load() == 1) {
        for (int64_t i0 = 0; i0 < items; i0 += (int64_t)1 << 30) {
            int64_t n = items - i0 < ((int64_t)1 << 30) ? items - i0 : ((int64_t)1 << 30);
            moba_attn_simt_kernel<<<(unsigned)n, 128, 0, st>>>(a, i0);
            count_launch();
        }
        return launch_ok();
    }
    const int rc = run_attention_tc(a, st);
    if (rc == MOBA_ERR_CUDA) {
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) cuda_fail(e);
    }
    if (rc == MOBA_OK && items > 0) count_launch();
    return rc;
}

template <bool VALIDATE, int NB>
int launch_merge(const Plan& P, const int32_t* idx, char* ws, void* out, float* lse, cudaStream_t st) {
    int64_t nrows = (int64_t)P.B * P.Hq * P.N;
    int dev = 0, nsm = 148, per_sm = 1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess)
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, moba_merge_kernel<VALIDATE, NB>, MERGE_THREADS, 0);
    if (e != cudaSuccess) return cuda_fail(e);
    int64_t grid = (int64_t)nsm * (per_sm > 0 ? per_sm : 1);
    const int64_t need = cdiv(nrows, MERGE_THREADS / 16);
    if (grid > need) grid = need;
    moba_merge_kernel<VALIDATE, NB><<<(unsigned)grid, MERGE_THREADS, 0, st>>>(
        idx, (const uint16_t*)(ws + P.off_opart), (const float*)(ws + P.off_lpart), (uint16_t*)out, lse, P.N, P.Hq,
        P.bs, P.topk, nrows);
    count_launch();
    return launch_ok();
}

template <bool VALIDATE>
int launch_merge_nb(const Plan& P, const int32_t* idx, char* ws, void* out, float* lse, cudaStream_t st) {
    if (P.kp <= 4) return launch_merge<VALIDATE, 4>(P, idx, ws, out, lse, st);
    if (P.kp <= 8) return launch_merge<VALIDATE, 8>(P, idx, ws, out, lse, st);
    if (P.kp <= 12) return launch_merge<VALIDATE, 12>(P, idx, ws, out, lse, st);
    return launch_merge<VALIDATE, 16>(P, idx, ws, out, lse, st);
}

// `validate`: the selection was given by the caller and is checked row by row; the gate's own
// selections are well formed by construction.
int run_merge(const Plan& P, const int32_t* idx, bool validate, char* ws, void* out, float* lse,
              cudaStream_t st) {
    return validate ? launch_merge_nb<true>(P, idx, ws, out, lse, st) : launch_merge_nb<false>(P, idx, ws, out, lse, st);
}

int forward_impl(const void* q, const void* k, const void* v, const int32_t* idx_in, void* out, float* lse,
                 int B, int Hq, int Hkv, int64_t N, int d, int bs, int topk, void* ws_ptr, size_t ws_bytes,
                 cudaStream_t st, PoolMode pm = PoolMode{0, nullptr}) {
    Plan P;
    int rc = make_plan(B, Hq, Hkv, N, d, bs, topk, &P);
    if (rc) return rc;
    if ((rc = check_ptrs({q, k, v, out, lse}))) return rc;
    if (idx_in && !aligned16(idx_in)) return MOBA_ERR_ALIGN;
    if ((rc = check_device())) return rc;
    bool own = false;
    char* ws = (char*)ws_ptr;
    if (!ws) {
        if (cudaMallocAsync((void**)&ws, P.total, st) != cudaSuccess) {
            cudaGetLastError();
            return MOBA_ERR_OOM;
        }
        own = true;
    } else if (ws_bytes < P.total || ((uintptr_t)ws & 255)) {
        return MOBA_ERR_WORKSPACE;
    }
    const int32_t* idx = idx_in;
    StageTimer timer(st);
    int done = 0;
    do {
        if (!idx) {
            int32_t* widx = (int32_t*)(ws + P.off_idx);
            const GateScratch gs = gate_scratch(P, ws, use_tc_gate(P));
            if ((rc = run_pool(P, k, gs, pm, st))) break;
            timer.mark(done++);
            if ((rc = run_gate(P, q, gs, widx, st))) break;
            timer.mark(done++);
            idx = widx;
        } else {
            timer.mark(done++);
            timer.mark(done++);
        }
        if ((rc = run_invert(P, idx, ws, st))) break;
        timer.mark(done++);
        AttnParams a = attn_params(P, q, k, v, out, lse, ws);
        if ((rc = run_attention(P, a, st))) break;
        timer.mark(done++);
        if ((rc = run_merge(P, idx, idx_in != nullptr, ws, out, lse, st))) break;
        timer.mark(done++);
    } while (0);
    timer.finish(done);
    if (own) cudaFreeAsync(ws, st);
    return rc;
}

// Options of the extended entry points; NULL means the defaults.
int parse_options(const moba_options* o, PoolMode* pm, bool* full) {
    *pm = PoolMode{0, nullptr};
    *full = false;
    if (!o) return MOBA_OK;
    if (o->struct_size < sizeof(moba_options) || o->reserved != 0) return MOBA_ERR_SHAPE;
    if (o->pooling < MOBA_POOL_MEAN || o->pooling > MOBA_POOL_WEIGHTED) return MOBA_ERR_SHAPE;
    if (o->pooling == MOBA_POOL_WEIGHTED && (!o->pool_weights || !aligned16(o->pool_weights))) return MOBA_ERR_SHAPE;
    if (o->full_attention != 0 && o->full_attention != 1) return MOBA_ERR_SHAPE;
    pm->mode = o->pooling;
    pm->w = o->pooling == MOBA_POOL_WEIGHTED ? o->pool_weights : nullptr;
    *full = o->full_attention == 1;
    return MOBA_OK;
}

int dense_impl(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq, int Hkv, int64_t N,
               int d, cudaStream_t st) {
    Plan P;
    if (N < 1 || N >= ((int64_t)1 << 31)) return MOBA_ERR_SHAPE;
    int rc = make_plan(B, Hq, Hkv, N, d, (int)N, 1, &P);
    if (rc) return rc;
    if ((rc = check_ptrs({q, k, v, out, lse}))) return rc;
    if ((rc = check_device())) return rc;
    AttnParams a = attn_params(P, q, k, v, out, lse, nullptr);
    a.dense = 1;
    a.Pmax = 0;
    a.L = 0;
    return run_attention(P, a, st);
}

}  // namespace

extern "C" {

const char* moba_status_string(int s) {
    switch (s) {
        case MOBA_OK: return "ok";
        case MOBA_ERR_NULL: return "null pointer";
        case MOBA_ERR_SHAPE: return "unsupported sizes";
        case MOBA_ERR_ALIGN: return "pointer not 16-byte aligned";
        case MOBA_ERR_UNSUPPORTED: return "device is not sm_100";
        case MOBA_ERR_CUDA: return "CUDA error";
        case MOBA_ERR_OOM: return "workspace allocation failed";
        case MOBA_ERR_DEVICE_TIMEOUT: return "device wait reached its limit";
        case MOBA_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
        case MOBA_ERR_SELECTION: return "malformed selection row";
        case MOBA_ERR_VALUE: return "invalid argument values (pooling weights)";
        default: return "unknown status";
    }
}

int moba_workspace_size(int B, int Hq, int Hkv, int64_t N, int d, int block_size, int topk, size_t* bytes) {
    if (!bytes) return MOBA_ERR_NULL;
    Plan P;
    int rc = make_plan(B, Hq, Hkv, N, d, block_size, topk, &P);
    if (rc) return rc;
    *bytes = P.total;
    return MOBA_OK;
}

int moba_forward(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq, int Hkv,
                 int64_t N, int d, int block_size, int topk, moba_stream_t stream) {
    return forward_impl(q, k, v, nullptr, out, lse, B, Hq, Hkv, N, d, block_size, topk, nullptr, 0,
                        (cudaStream_t)stream);
}

int moba_forward_ws(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq, int Hkv,
                    int64_t N, int d, int block_size, int topk, void* workspace, size_t workspace_bytes,
                    moba_stream_t stream) {
    if (!workspace) return MOBA_ERR_WORKSPACE;
    return forward_impl(q, k, v, nullptr, out, lse, B, Hq, Hkv, N, d, block_size, topk, workspace,
                        workspace_bytes, (cudaStream_t)stream);
}

int moba_forward_selected(const void* q, const void* k, const void* v, const int32_t* idx, void* out, float* lse,
                          int B, int Hq, int Hkv, int64_t N, int d, int block_size, int topk,
                          moba_stream_t stream) {
    if (!idx) return MOBA_ERR_NULL;
    return forward_impl(q, k, v, idx, out, lse, B, Hq, Hkv, N, d, block_size, topk, nullptr, 0,
                        (cudaStream_t)stream);
}

int moba_forward_selected_ws(const void* q, const void* k, const void* v, const int32_t* idx, void* out,
                             float* lse, int B, int Hq, int Hkv, int64_t N, int d, int block_size, int topk,
                             void* workspace, size_t workspace_bytes, moba_stream_t stream) {
    if (!idx) return MOBA_ERR_NULL;
    if (!workspace) return MOBA_ERR_WORKSPACE;
    return forward_impl(q, k, v, idx, out, lse, B, Hq, Hkv, N, d, block_size, topk, workspace, workspace_bytes,
                        (cudaStream_t)stream);
}

int moba_gate(const void* q, const void* k, int32_t* idx, int B, int Hq, int Hkv, int64_t N, int d,
              int block_size, int topk, moba_stream_t stream) {
    Plan P;
    int rc = make_plan(B, Hq, Hkv, N, d, block_size, topk, &P);
    if (rc) return rc;
    if ((rc = check_ptrs({q, k, (const void*)idx}))) return rc;
    if ((rc = check_device())) return rc;
    cudaStream_t st = (cudaStream_t)stream;
    char* scratch = nullptr;
    if (cudaMallocAsync((void**)&scratch, P.gate_bytes, st) != cudaSuccess) {
        cudaGetLastError();
        return MOBA_ERR_OOM;
    }
    const GateScratch gs = gate_scratch(P, scratch, use_tc_gate(P));
    rc = run_pool(P, k, gs, PoolMode{0, nullptr}, st);
    if (!rc) rc = run_gate(P, q, gs, idx, st);
    cudaFreeAsync(scratch, st);
    return rc;
}

int moba_dense_causal(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq, int Hkv,
                      int64_t N, int d, moba_stream_t stream) {
    return dense_impl(q, k, v, out, lse, B, Hq, Hkv, N, d, (cudaStream_t)stream);
}

int moba_forward_ex(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq, int Hkv,
                    int64_t N, int d, int block_size, int topk, const moba_options* options, void* workspace,
                    size_t workspace_bytes, moba_stream_t stream) {
    PoolMode pm;
    bool full = false;
    int rc = parse_options(options, &pm, &full);
    if (rc) return rc;
    if (full) {  // a full-attention layer of a hybrid model
        Plan P;
        if ((rc = make_plan(B, Hq, Hkv, N, d, block_size, topk, &P))) return rc;
        return dense_impl(q, k, v, out, lse, B, Hq, Hkv, N, d, (cudaStream_t)stream);
    }
    return forward_impl(q, k, v, nullptr, out, lse, B, Hq, Hkv, N, d, block_size, topk, workspace, workspace_bytes,
                        (cudaStream_t)stream, pm);
}

int moba_gate_ex(const void* q, const void* k, int32_t* idx, int B, int Hq, int Hkv, int64_t N, int d,
                 int block_size, int topk, const moba_options* options, moba_stream_t stream) {
    PoolMode pm;
    bool full = false;
    int rc = parse_options(options, &pm, &full);
    if (rc) return rc;
    if (full) return MOBA_ERR_SHAPE;  // a full-attention layer has no gate
    Plan P;
    if ((rc = make_plan(B, Hq, Hkv, N, d, block_size, topk, &P))) return rc;
    if ((rc = check_ptrs({q, k, (const void*)idx}))) return rc;
    if ((rc = check_device())) return rc;
    cudaStream_t st = (cudaStream_t)stream;
    char* scratch = nullptr;
    if (cudaMallocAsync((void**)&scratch, P.gate_bytes, st) != cudaSuccess) {
        cudaGetLastError();
        return MOBA_ERR_OOM;
    }
    const GateScratch gs = gate_scratch(P, scratch, use_tc_gate(P));
    rc = run_pool(P, k, gs, pm, st);
    if (!rc) rc = run_gate(P, q, gs, idx, st);
    cudaFreeAsync(scratch, st);
    return rc;
}

int moba_sync_status(moba_stream_t stream) {
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e);
    int flag = 0;
    if ((e = cudaMemcpyFromSymbol(&flag, g_moba_err, sizeof(int))) != cudaSuccess) return cuda_fail(e);
    if (flag) {
        int zero = 0;
        if ((e = cudaMemcpyToSymbol(g_moba_err, &zero, sizeof(int))) != cudaSuccess) return cuda_fail(e);
    }
    return flag;
}

int moba_selftest_wait_timeout(int64_t limit_ns, moba_stream_t stream) {
    if (limit_ns < 1000 || limit_ns > 10000000000LL) return MOBA_ERR_SHAPE;
    int rc = check_device();
    if (rc) return rc;
    moba_wait_selftest_kernel<<<1, 32, 0, (cudaStream_t)stream>>>((uint64_t)limit_ns);
    count_launch();
    return launch_ok();
}

int moba_stage_timing(int enable) {
    std::lock_guard<std::mutex> lk(g_timing_mu);
    int old = g_timing ? 1 : 0;
    g_timing = enable != 0;
    return old;
}

int moba_stage_times(float* ms, int n, int* calls) {
    if (!ms || n < 1) return MOBA_ERR_NULL;
    std::vector<StageRec> recs;
    {
        std::lock_guard<std::mutex> lk(g_timing_mu);
        recs.swap(g_recs);
    }
    for (int i = 0; i < n; ++i) ms[i] = 0.f;
    int rc = MOBA_OK;
    for (auto& r : recs) {
        if (cudaEventSynchronize(r.ev[kStages]) != cudaSuccess) rc = MOBA_ERR_CUDA;
        for (int i = 0; i < kStages && i < n; ++i) {
            float t = 0.f;
            if (rc == MOBA_OK && cudaEventElapsedTime(&t, r.ev[i], r.ev[i + 1]) == cudaSuccess) ms[i] += t;
        }
        for (int i = 0; i <= kStages; ++i) cudaEventDestroy(r.ev[i]);
    }
    if (calls) *calls = (int)recs.size();
    if (rc != MOBA_OK) cudaGetLastError();
    return rc;
}

uint64_t moba_launch_count(void) { return g_launches.load(); }

const char* moba_last_error_string(void) { return g_last_cuda_error; }

int moba_set_attention_impl(int impl) {
    if (impl != 0 && impl != 1) return MOBA_ERR_SHAPE;
    return g_attn_impl.exchange(impl);
}

int moba_set_gate_impl(int impl) {
    if (impl != 0 && impl != 1) return MOBA_ERR_SHAPE;
    return g_gate_impl.exchange(impl);
}

}  // extern "C"

// ---------------------------------------------------------------- backward
namespace {

// The forward plan's gate scratch, selection and inversion arrays, then D, the fp32 dq
// accumulator and the work counter (the forward's partials are not needed).
struct BwdPlan {
    Plan P;
    size_t off_D, off_acc, off_counter, total;
};

int make_bwd_plan(int B, int Hq, int Hkv, int64_t N, int d, int bs, int topk, BwdPlan* bp) {
    int rc = make_plan(B, Hq, Hkv, N, d, bs, topk, &bp->P);
    if (rc) return rc;
    size_t o = bp->P.off_opart;  // everything before the partials
    bp->off_D = o;
    o = align256(o + sizeof(float) * (size_t)B * Hq * N);
    bp->off_acc = o;
    o = align256(o + sizeof(float) * (size_t)B * N * Hq * MOBA_D);
    bp->off_counter = o;
    o = align256(o + sizeof(int));
    bp->total = o;
    return MOBA_OK;
}

}  // namespace

extern "C" int moba_backward_workspace_size(int B, int Hq, int Hkv, int64_t N, int d, int block_size, int topk,
                                            size_t* bytes) {
    if (!bytes) return MOBA_ERR_NULL;
    BwdPlan bp;
    const int rc = make_bwd_plan(B, Hq, Hkv, N, d, block_size, topk, &bp);
    if (rc) return rc;
    *bytes = bp.total;
    return MOBA_OK;
}

extern "C" int moba_backward(const void* q, const void* k, const void* v, const void* out, const float* lse,
                             const void* dout, const int32_t* idx, void* dq, void* dk, void* dv, int B, int Hq, int Hkv,
                             int64_t N, int d, int block_size, int topk, void* workspace, size_t workspace_bytes,
                             moba_stream_t stream) {
    BwdPlan bp;
    int rc = make_bwd_plan(B, Hq, Hkv, N, d, block_size, topk, &bp);
    if (rc) return rc;
    const Plan& P = bp.P;
    if ((rc = check_ptrs({q, k, v, out, (const void*)lse, dout, dq, dk, dv}))) return rc;
    if (idx && !aligned16(idx)) return MOBA_ERR_ALIGN;
    if ((rc = check_device())) return rc;
    cudaStream_t st = (cudaStream_t)stream;
    bool own = false;
    char* ws = (char*)workspace;
    if (!ws) {
        if (cudaMallocAsync((void**)&ws, bp.total, st) != cudaSuccess) {
            cudaGetLastError();
            return MOBA_ERR_OOM;
        }
        own = true;
    } else if (workspace_bytes < bp.total || ((uintptr_t)ws & 255)) {
        return MOBA_ERR_WORKSPACE;
    }
    do {
        // the selection: the caller's (checked row by row by the inversion), or the gate's again
        const int32_t* sel = idx;
        if (!sel) {
            int32_t* widx = (int32_t*)(ws + P.off_idx);
            const GateScratch gs = gate_scratch(P, ws, use_tc_gate(P));
            if ((rc = run_pool(P, k, gs, PoolMode{0, nullptr}, st))) break;
            if ((rc = run_gate(P, q, gs, widx, st))) break;
            sel = widx;
        }
        if ((rc = run_invert(P, sel, ws, st))) break;
        float* D = (float*)(ws + bp.off_D);
        float* acc = (float*)(ws + bp.off_acc);
        int* counter = (int*)(ws + bp.off_counter);
        const int64_t nrows = (int64_t)B * Hq * N;
        moba_bwd_prep_kernel<<<(unsigned)cdiv(nrows * 16, 256), 256, 0, st>>>((const uint16_t*)out,
                                                                              (const uint16_t*)dout, D, N, Hq, nrows);
        count_launch();
        if ((rc = launch_ok())) break;
        cudaError_t e = cudaMemsetAsync(acc, 0, sizeof(float) * (size_t)B * N * Hq * MOBA_D, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(counter, 0, sizeof(int), st);
        if (e != cudaSuccess) {
            rc = cuda_fail(e);
            break;
        }
        BwdParams bpar;
        bpar.q = (const uint16_t*)q;
        bpar.dout = (const uint16_t*)dout;
        bpar.lse = lse;
        bpar.Dvec = D;
        bpar.dk = (uint16_t*)dk;
        bpar.dv = (uint16_t*)dv;
        bpar.dq_acc = acc;
        bpar.entries = (const uint64_t*)(ws + P.off_entries);
        bpar.segoff = (const int64_t*)(ws + P.off_segoff);
        bpar.counter = counter;
        bpar.N = N;
        bpar.nblk = P.nblk;
        bpar.nch = P.nch;
        bpar.mb = P.mb;
        bpar.items = P.L * P.mb;
        bpar.B = B;
        bpar.Hq = Hq;
        bpar.Hkv = Hkv;
        bpar.G = P.G;
        bpar.bs = block_size;
        bpar.scale_log2 = (float)(1.4426950408889634 / sqrt((double)d));
        bpar.scale = (float)(1.0 / sqrt((double)d));
        TcMaps maps;
        if (!moba_make_kv_map(&maps.k, k, (int64_t)B * N, Hkv) || !moba_make_kv_map(&maps.v, v, (int64_t)B * N, Hkv)) {
            rc = MOBA_ERR_CUDA;
            break;
        }
        int dev = 0, nsm = 0;
        if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
            (e = cudaFuncSetAttribute(moba_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      BWD_SMEM_BYTES)) != cudaSuccess) {
            rc = cuda_fail(e);
            break;
        }
        const int64_t grid = bpar.items < nsm ? bpar.items : nsm;
        moba_bwd_kernel<<<(unsigned)grid, BWD_THREADS, BWD_SMEM_BYTES, st>>>(bpar, maps);
        count_launch();
        if ((rc = launch_ok())) break;
        const int64_t n4 = (int64_t)B * N * Hq * MOBA_D / 4;
        moba_bwd_dq_kernel<<<(unsigned)cdiv(n4, 256), 256, 0, st>>>(acc, (uint16_t*)dq, bpar.scale, n4);
        count_launch();
        rc = launch_ok();
    } while (0);
    if (own) cudaFreeAsync(ws, st);
    return rc;
}

// ---------------------------------------------------------------- packed (varlen) batches
// Each packed sequence is its own context. Consecutive sequences of equal length are one
// batched call of the fixed-length path (their tokens are adjacent, so [n, len, H, d] is a view of
// the packed [total, H, d]); lse and idx, packed as [Hq, total(, topk)], are written through a
// buffer in the workspace and one strided 2-D copy per sequence.
namespace {

struct VarRun {
    int64_t s0, n, len, tok0;  // first sequence, sequences, their length, first token
};

int varlen_runs(const int64_t* cu, int nseq, std::vector<VarRun>* runs, int64_t* total) {
    if (!cu) return MOBA_ERR_NULL;
    if (nseq < 1 || cu[0] != 0) return MOBA_ERR_SHAPE;
    runs->clear();
    for (int s = 0; s < nseq; ++s) {
        const int64_t len = cu[s + 1] - cu[s];
        if (len < 0) return MOBA_ERR_SHAPE;
        if (len == 0) continue;
        if (!runs->empty() && runs->back().len == len && runs->back().s0 + runs->back().n == s &&
            runs->back().n < 65535)
            runs->back().n += 1;
        else
            runs->push_back(VarRun{s, 1, len, cu[s]});
    }
    *total = cu[nseq];
    if (*total >= ((int64_t)1 << 31)) return MOBA_ERR_SHAPE;
    return MOBA_OK;
}

// Workspace of the varlen entry points: the largest run's forward workspace (or gate scratch plus
// its selection), then the largest run's lse / idx staging buffer.
int varlen_plan(const std::vector<VarRun>& runs, int Hq, int Hkv, int d, int bs, int topk, size_t* fwd,
                size_t* stage, size_t* total) {
    *fwd = 0;
    *stage = 0;
    for (const VarRun& r : runs) {
        Plan P;
        const int rc = make_plan((int)r.n, Hq, Hkv, r.len, d, bs, topk, &P);
        if (rc) return rc;
        const size_t gate_need = P.gate_bytes;  // the gate path keeps its selection in the staging buffer
        *fwd = *fwd > P.total ? *fwd : P.total;
        *fwd = *fwd > gate_need ? *fwd : gate_need;
        const size_t st_lse = sizeof(float) * (size_t)(r.n * Hq * r.len);
        const size_t st_idx = sizeof(int32_t) * (size_t)(r.n * Hq * r.len * topk);
        const size_t need = st_lse > st_idx ? st_lse : st_idx;
        *stage = *stage > need ? *stage : need;
    }
    *total = align256(*fwd) + align256(*stage > 0 ? *stage : 1);
    return MOBA_OK;
}

// dst[h][tok0 + b*len + t] (row pitch total) <- src[b][h][t] for every sequence b of the run
int varlen_scatter(void* dst, const void* src, const VarRun& r, int Hq, int64_t total, size_t elem, cudaStream_t st) {
    for (int64_t b = 0; b < r.n; ++b) {
        const char* s = (const char*)src + (size_t)(b * Hq * r.len) * elem;
        char* dd = (char*)dst + (size_t)(r.tok0 + b * r.len) * elem;
        const cudaError_t e = cudaMemcpy2DAsync(dd, (size_t)total * elem, s, (size_t)r.len * elem,
                                                (size_t)r.len * elem, (size_t)Hq, cudaMemcpyDeviceToDevice, st);
        if (e != cudaSuccess) return cuda_fail(e);
    }
    return MOBA_OK;
}

}  // namespace

extern "C" int moba_varlen_workspace_size(const int64_t* cu_seqlens, int nseq, int Hq, int Hkv, int d, int block_size,
                                          int topk, size_t* bytes) {
    if (!bytes) return MOBA_ERR_NULL;
    std::vector<VarRun> runs;
    int64_t total = 0;
    int rc = varlen_runs(cu_seqlens, nseq, &runs, &total);
    if (rc) return rc;
    size_t fwd, stage;
    if ((rc = varlen_plan(runs, Hq, Hkv, d, block_size, topk, &fwd, &stage, bytes))) return rc;
    return MOBA_OK;
}

extern "C" int moba_forward_varlen(const void* q, const void* k, const void* v, void* out, float* lse,
                                   const int64_t* cu_seqlens, int nseq, int Hq, int Hkv, int d, int block_size,
                                   int topk, const moba_options* options, void* workspace, size_t workspace_bytes,
                                   moba_stream_t stream) {
    std::vector<VarRun> runs;
    int64_t total = 0;
    int rc = varlen_runs(cu_seqlens, nseq, &runs, &total);
    if (rc) return rc;
    size_t fwd, stage, need;
    if ((rc = varlen_plan(runs, Hq, Hkv, d, block_size, topk, &fwd, &stage, &need))) return rc;
    PoolMode pm;
    bool full = false;
    if ((rc = parse_options(options, &pm, &full))) return rc;
    if ((rc = check_ptrs({q, k, v, out, (const void*)lse}))) return rc;
    if ((rc = check_device())) return rc;
    cudaStream_t st = (cudaStream_t)stream;
    bool own = false;
    char* ws = (char*)workspace;
    if (!ws) {
        if (cudaMallocAsync((void**)&ws, need, st) != cudaSuccess) {
            cudaGetLastError();
            return MOBA_ERR_OOM;
        }
        own = true;
    } else if (workspace_bytes < need || ((uintptr_t)ws & 255)) {
        return MOBA_ERR_WORKSPACE;
    }
    float* lse_stage = (float*)(ws + align256(fwd));
    for (const VarRun& r : runs) {
        const size_t qoff = (size_t)r.tok0 * Hq * MOBA_D, koff = (size_t)r.tok0 * Hkv * MOBA_D;
        const uint16_t* qr = (const uint16_t*)q + qoff;
        const uint16_t* kr = (const uint16_t*)k + koff;
        const uint16_t* vr = (const uint16_t*)v + koff;
        uint16_t* orr = (uint16_t*)out + qoff;
        if (full)
            rc = dense_impl(qr, kr, vr, orr, lse_stage, (int)r.n, Hq, Hkv, r.len, d, st);
        else
            rc = forward_impl(qr, kr, vr, nullptr, orr, lse_stage, (int)r.n, Hq, Hkv, r.len, d, block_size, topk, ws,
                              fwd, st, pm);
        if (rc) break;
        if ((rc = varlen_scatter(lse, lse_stage, r, Hq, total, sizeof(float), st))) break;
    }
    if (own) cudaFreeAsync(ws, st);
    return rc;
}

extern "C" int moba_gate_varlen(const void* q, const void* k, int32_t* idx, const int64_t* cu_seqlens, int nseq, int Hq,
                                int Hkv, int d, int block_size, int topk, const moba_options* options, void* workspace,
                                size_t workspace_bytes, moba_stream_t stream) {
    std::vector<VarRun> runs;
    int64_t total = 0;
    int rc = varlen_runs(cu_seqlens, nseq, &runs, &total);
    if (rc) return rc;
    size_t fwd, stage, need;
    if ((rc = varlen_plan(runs, Hq, Hkv, d, block_size, topk, &fwd, &stage, &need))) return rc;
    PoolMode pm;
    bool full = false;
    if ((rc = parse_options(options, &pm, &full))) return rc;
    if (full) return MOBA_ERR_SHAPE;
    if ((rc = check_ptrs({q, k, (const void*)idx}))) return rc;
    if ((rc = check_device())) return rc;
    cudaStream_t st = (cudaStream_t)stream;
    bool own = false;
    char* ws = (char*)workspace;
    if (!ws) {
        if (cudaMallocAsync((void**)&ws, need, st) != cudaSuccess) {
            cudaGetLastError();
            return MOBA_ERR_OOM;
        }
        own = true;
    } else if (workspace_bytes < need || ((uintptr_t)ws & 255)) {
        return MOBA_ERR_WORKSPACE;
    }
    int32_t* idx_stage = (int32_t*)(ws + align256(fwd));
    for (const VarRun& r : runs) {
        Plan P;
        if ((rc = make_plan((int)r.n, Hq, Hkv, r.len, d, block_size, topk, &P))) break;
        const GateScratch gs = gate_scratch(P, ws, use_tc_gate(P));
        const uint16_t* qr = (const uint16_t*)q + (size_t)r.tok0 * Hq * MOBA_D;
        const uint16_t* kr = (const uint16_t*)k + (size_t)r.tok0 * Hkv * MOBA_D;
        if ((rc = run_pool(P, kr, gs, pm, st))) break;
        if ((rc = run_gate(P, qr, gs, idx_stage, st))) break;
        if ((rc = varlen_scatter(idx, idx_stage, r, Hq, total, sizeof(int32_t) * topk, st))) break;
    }
    if (own) cudaFreeAsync(ws, st);
    return rc;
}

// ---------------------------------------------------------------- decode step
namespace {

struct DecodePlan {
    int64_t c, umax, chunk, nch, nfull_needed;
    size_t off_kept, off_count, off_list, off_mask, off_part, total;
};

int make_decode_plan(int B, int Hq, int Hkv, int64_t L, int d, int bs, int topk, int full, DecodePlan* dp) {
    if (B < 1 || Hq < 1 || Hkv < 1 || L < 1 || bs < 1 || topk < 1 || d != MOBA_D || Hq % Hkv != 0) return MOBA_ERR_SHAPE;
    if (topk > MOBA_MAX_TOPK || Hq / Hkv > DEC_MAX_G || (full != 0 && full != 1)) return MOBA_ERR_SHAPE;
    if (B > 65535 || Hkv > 65535 || L >= ((int64_t)1 << 31) || cdiv(L, bs) > MOBA_MAX_BLOCKS) return MOBA_ERR_SHAPE;
    const int G = Hq / Hkv;
    dp->c = (L - 1) / bs;
    dp->nfull_needed = dp->c;  // summaries of the earlier blocks 0 .. c - 1
    const int64_t kp = topk - 1;
    const int64_t past = full ? dp->c : (dp->c < (int64_t)G * kp ? dp->c : (int64_t)G * kp);
    dp->umax = past + 1;
    // keys per attend CTA: 512, doubled (up to 4096, not past the block) while the grid keeps at
    // least 8 CTAs per SM, so that long unions run fewer, longer CTAs (each pays its pipeline
    // fill and combine once) with fewer partials to merge
    int nsm = 148;
    {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || nsm < 1) {
            cudaGetLastError();
            nsm = 148;
        }
    }
    dp->chunk = DEC_MIN_CHUNK;
    while (dp->chunk < 4096 && dp->chunk < bs &&
           (int64_t)B * Hkv * dp->umax * cdiv(bs, 2 * dp->chunk) >= 8 * (int64_t)nsm)
        dp->chunk *= 2;
    dp->nch = cdiv(bs, dp->chunk);
    const int64_t units = (int64_t)B * Hkv;
    size_t o = 0;
    dp->off_kept = o;
    o = align256(o + sizeof(int32_t) * (size_t)(units * G * (kp > 0 ? kp : 1)));
    dp->off_count = o;
    o = align256(o + sizeof(int32_t) * (size_t)units);
    dp->off_list = o;
    o = align256(o + sizeof(int32_t) * (size_t)(units * dp->umax));
    dp->off_mask = o;
    o = align256(o + sizeof(uint32_t) * (size_t)(units * dp->umax));
    dp->off_part = o;
    o = align256(o + sizeof(float) * (size_t)(units * dp->umax * dp->nch * G * DEC_PART));
    dp->total = o;
    return MOBA_OK;
}


// Launch of a decode kernel as a programmatic dependent of the kernel before it on the stream:
// its CTAs may start while that kernel finishes, and wait for its results in griddepcontrol.wait.
template <typename Kernel>
cudaError_t launch_dependent(Kernel kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                             const DecodeParams& p) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, p);
}

}  // namespace

extern "C" int moba_decode_workspace_size(int B, int Hq, int Hkv, int64_t L, int d, int block_size, int topk,
                                          int full_attention, size_t* bytes) {
    if (!bytes) return MOBA_ERR_NULL;
    DecodePlan dp;
    const int rc = make_decode_plan(B, Hq, Hkv, L, d, block_size, topk, full_attention, &dp);
    if (rc) return rc;
    *bytes = dp.total;
    return MOBA_OK;
}

extern "C" int moba_pool_cache(const void* k, double* kbar, int B, int Hkv, int64_t L, int64_t Lmax, int d,
                               int block_size, int64_t kbar_rows, int64_t first_block, const moba_options* options,
                               moba_stream_t stream) {
    if (B < 1 || Hkv < 1 || L < 0 || Lmax < L || d != MOBA_D || block_size < 1 || first_block < 0) return MOBA_ERR_SHAPE;
    if (B > 65535 || Hkv > 65535 || Lmax >= ((int64_t)1 << 31) || (int64_t)B * Lmax >= ((int64_t)1 << 31))
        return MOBA_ERR_SHAPE;
    const int64_t nfull = L / block_size;
    if (kbar_rows < nfull) return MOBA_ERR_SHAPE;
    int rc = check_ptrs({k, (const void*)kbar});
    if (rc) return rc;
    PoolMode pm;
    bool full = false;
    if ((rc = parse_options(options, &pm, &full))) return rc;
    if ((rc = check_device())) return rc;
    if (first_block >= nfull) return MOBA_OK;  // nothing newly full
    pm.j0 = first_block;
    pm.rows = kbar_rows;
    dim3 grid((unsigned)(nfull - first_block), Hkv, B);
    moba_pool_kernel<<<grid, POOL_THREADS, 0, (cudaStream_t)stream>>>((const uint16_t*)k, kbar, Lmax, Hkv, block_size,
                                                                        nfull, PoolAux{nullptr, nullptr, nullptr}, pm);
    count_launch();
    return launch_ok();
}

extern "C" int moba_decode(const void* q, const void* k, const void* v, const double* kbar, int64_t kbar_rows,
                           void* out, float* lse, int32_t* idx, int B, int Hq, int Hkv, int64_t L, int64_t Lmax, int d,
                           int block_size, int topk, int full_attention, void* workspace, size_t workspace_bytes,
                           moba_stream_t stream) {
    DecodePlan dp;
    int rc = make_decode_plan(B, Hq, Hkv, L, d, block_size, topk, full_attention, &dp);
    if (rc) return rc;
    if (Lmax < L || (int64_t)B * Lmax >= ((int64_t)1 << 31)) return MOBA_ERR_SHAPE;
    if (!full_attention && kbar_rows < dp.nfull_needed) return MOBA_ERR_SHAPE;
    if ((rc = check_ptrs({q, k, v, out, (const void*)lse}))) return rc;
    if (!full_attention && dp.c > 0 && !kbar) return MOBA_ERR_NULL;
    if ((kbar && !aligned16(kbar)) || (idx && !aligned16(idx))) return MOBA_ERR_ALIGN;
    if ((rc = check_device())) return rc;
    cudaStream_t st = (cudaStream_t)stream;
    bool own = false;
    char* ws = (char*)workspace;
    if (!ws) {
        if (cudaMallocAsync((void**)&ws, dp.total, st) != cudaSuccess) {
            cudaGetLastError();
            return MOBA_ERR_OOM;
        }
        own = true;
    } else if (workspace_bytes < dp.total || ((uintptr_t)ws & 255)) {
        return MOBA_ERR_WORKSPACE;
    }
    DecodeParams p;
    p.q = (const uint16_t*)q;
    p.k = (const uint16_t*)k;
    p.v = (const uint16_t*)v;
    p.kbar = kbar;
    p.kbar_rows = kbar_rows;
    p.L = L;
    p.Lmax = Lmax;
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.G = Hq / Hkv;
    p.bs = block_size;
    p.topk = topk;
    p.c = dp.c;
    p.umax = dp.umax;
    p.chunk = dp.chunk;
    p.nch = dp.nch;
    p.full = full_attention;
    p.kept = (int32_t*)(ws + dp.off_kept);
    p.ucount = (int32_t*)(ws + dp.off_count);
    p.ulist = (int32_t*)(ws + dp.off_list);
    p.umask = (uint32_t*)(ws + dp.off_mask);
    p.part = (float*)(ws + dp.off_part);
    p.idx_out = full_attention ? nullptr : idx;
    p.out = (uint16_t*)out;
    p.lse = lse;
    p.scale_log2 = (float)(1.4426950408889634 / sqrt((double)d));
    do {
        const int kp = topk - 1;
        if (!full_attention && dp.c > kp && kp > 0) {  // otherwise no scores are needed
            const size_t smem_sel = sizeof(double) * (size_t)(dp.c + 2 * DEC_SEL_WARPS * kp) +
                                    sizeof(int32_t) * (size_t)(2 * DEC_SEL_WARPS * kp + dp.c);
            cudaError_t e = cudaFuncSetAttribute(moba_decode_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)smem_sel);
            if (e != cudaSuccess) {
                rc = cuda_fail(e);
                break;
            }
            moba_decode_select_kernel<<<dim3(p.G, Hkv, B), DEC_SEL_THREADS, smem_sel, st>>>(p);
        } else if (!full_attention) {
            moba_decode_select_kernel<<<dim3(p.G, Hkv, B), DEC_SEL_THREADS, 0, st>>>(p);
        }
        if (!full_attention) {
            count_launch();
            if ((rc = launch_ok())) break;
        }
        {
            const size_t smem_union = full_attention ? 0 : sizeof(uint32_t) * (size_t)(dp.c > 0 ? dp.c : 1);
            cudaError_t e = cudaFuncSetAttribute(moba_decode_union_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)smem_union);
            if (e != cudaSuccess) {
                rc = cuda_fail(e);
                break;
            }
            e = launch_dependent(moba_decode_union_kernel, dim3(Hkv, B), dim3(DEC_UNION_THREADS), smem_union, st, p);
            if (e != cudaSuccess) {
                rc = cuda_fail(e);
                break;
            }
            count_launch();
            if ((rc = launch_ok())) break;
        }
        {
            cudaError_t e = cudaFuncSetAttribute(moba_decode_attend_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 DEC_ATTEND_SMEM);
            if (e != cudaSuccess) {
                rc = cuda_fail(e);
                break;
            }
            dim3 grid((unsigned)(p.umax * p.nch), Hkv, B);
            e = launch_dependent(moba_decode_attend_kernel, grid, dim3(DEC_WARPS * 32), DEC_ATTEND_SMEM, st, p);
            if (e != cudaSuccess) {
                rc = cuda_fail(e);
                break;
            }
            count_launch();
            if ((rc = launch_ok())) break;
        }
        {
            const cudaError_t e = launch_dependent(moba_decode_merge_kernel, dim3(Hq, B), dim3(DEC_MERGE_THREADS), 0, st, p);
            if (e != cudaSuccess) {
                rc = cuda_fail(e);
                break;
            }
        }
        count_launch();
        rc = launch_ok();
    } while (0);
    if (own) cudaFreeAsync(ws, st);
    return rc;
}

// ---------------------------------------------------------------- allocation-free gate
// Some callers cannot allocate device memory while they run: serving engines
// that reserve nearly all HBM up front for their KV cache and hand out only
// pre-planned buffers (a cudaMallocAsync there either fails or breaks the plan),
// and embedders with a fixed, audited memory budget that forbids allocation
// inside a call. moba_gate_noalloc serves them: it runs the pooling kernel and
// the fp64 CUDA-core gate (the gate whose only scratch is the block means), and
// those block means live in the fixed array below instead of a stream-ordered
// allocation. Its selections are the ones moba_gate returns (both gates give
// the exact fp64 selection); at long sequences it is slower than moba_gate's
// default tensor-core gate.
//
// The array is part of the library image: every GPU that loads the library holds
// its 8 MiB until the process exits. In host code its name is only a host-side
// stand-in, so the device address is looked up with cudaGetSymbolAddress on the
// first call made with a device current (that first call should therefore come
// before any stream capture), and looked up again only when the calling thread's
// CUDA context is a different one than at the last lookup on that device (after a
// device reset, the module is loaded again at another address). All calls share
// the array and it keeps the last call's contents; the pooling kernel overwrites
// every entry the gate reads, so nothing needs clearing. Calls that overlap on the
// GPU (different streams, or different host threads, on the same device) race on it.
#define MOBA_NOALLOC_KBAR_ROWS 8192  // B * Hkv * floor(N / block_size) <= 8192 (8 MiB of doubles)
static __device__ __align__(256) double g_noalloc_kbar[MOBA_NOALLOC_KBAR_ROWS * MOBA_D];

namespace {
std::mutex g_noalloc_mu;
constexpr int kNoallocMaxDevices = 64;
struct NoallocSlot {
    double* ptr;
    unsigned long long ctx_id;
    bool have_id;
};
NoallocSlot g_noalloc_slot[kNoallocMaxDevices] = {};

typedef CUresult (*moba_ctx_get_current_fn)(CUcontext*);
typedef CUresult (*moba_ctx_get_id_fn)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current CUDA context (false when there is none yet,
// or when the driver does not offer the query).
bool current_ctx_id(unsigned long long* id) {
    static moba_ctx_get_current_fn get_cur = nullptr;
    static moba_ctx_get_id_fn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q;
        void* p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_cur = (moba_ctx_get_current_fn)p;
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = (moba_ctx_get_id_fn)p;
    });
    if (!get_cur || !get_id) return false;
    CUcontext ctx = nullptr;
    if (get_cur(&ctx) != CUDA_SUCCESS || !ctx) return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}
}  // namespace

extern "C" int moba_gate_noalloc(const void* q, const void* k, int32_t* idx, int B, int Hq, int Hkv, int64_t N,
                                 int d, int block_size, int topk, moba_stream_t stream) {
    Plan P;
    int rc = make_plan(B, Hq, Hkv, N, d, block_size, topk, &P);
    if (rc) return rc;
    if ((int64_t)B * Hkv * P.nfull > MOBA_NOALLOC_KBAR_ROWS) return MOBA_ERR_SHAPE;
    if ((rc = check_ptrs({q, k, (const void*)idx}))) return rc;
    if ((rc = check_device())) return rc;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev < 0 || dev >= kNoallocMaxDevices) return MOBA_ERR_UNSUPPORTED;
    double* kbar = nullptr;
    {
        std::lock_guard<std::mutex> lk(g_noalloc_mu);
        NoallocSlot& slot = g_noalloc_slot[dev];
        unsigned long long ctx = 0;
        const bool have = current_ctx_id(&ctx);
        if (!slot.ptr || !have || !slot.have_id || slot.ctx_id != ctx) {
            void* p = nullptr;
            if ((e = cudaGetSymbolAddress(&p, g_noalloc_kbar)) != cudaSuccess) return cuda_fail(e);
            if (!p) return MOBA_ERR_CUDA;
            slot.ptr = (double*)p;
            slot.have_id = current_ctx_id(&slot.ctx_id);  // the lookup made the context current
        }
        kbar = slot.ptr;
    }
    cudaStream_t st = (cudaStream_t)stream;
    GateScratch gs;
    gs.kbar = kbar;
    gs.aux = PoolAux{nullptr, nullptr, nullptr};  // the fp64 gate: its only scratch is Kbar
    rc = run_pool(P, k, gs, PoolMode{0, nullptr}, st);
    if (!rc) rc = run_gate(P, q, gs, idx, st);
    return rc;
}

#ifdef MOBA_GATE_STATS
extern "C" int moba_debug_gate_stats(unsigned long long* out4, int reset) {
    if (cudaMemcpyFromSymbol(out4, g_gate_stats, sizeof(unsigned long long) * 4) != cudaSuccess) return MOBA_ERR_CUDA;
    if (reset) {
        unsigned long long z[4] = {0, 0, 0, 0};
        if (cudaMemcpyToSymbol(g_gate_stats, z, sizeof(z)) != cudaSuccess) return MOBA_ERR_CUDA;
    }
    return MOBA_OK;
}
#endif

