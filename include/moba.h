/*
 * moba.h - C ABI of libmoba, the sm_100a (B200) implementation of the causal
 * prefill forward of MoBA (Mixture of Block Attention).
 *
 * The method (sources: "MoBA project hub" page, Steps 1-3; "MoBA tech-report
 * summary" page, section 2; "KIMI MoBA" blog, section 3 configuration fields;
 * "NSA vs MoBA" blog, section 1 attention formula):
 *   - keys are cut into blocks of block_size consecutive tokens; token t lies
 *     in block c(t) = floor(t / block_size);
 *   - each full block j is represented by the mean of its keys, Kbar_j;
 *   - query t scores every earlier block j < c(t) as <q_t, Kbar_j> (no gate
 *     parameters, no scaling), always keeps its own block c(t), and keeps the
 *     topk - 1 best earlier blocks (higher score first, lower block index on
 *     equal scores); with c(t) <= topk - 1 every earlier block is kept;
 *   - it attends with softmax(q k^T / sqrt(d)) over all keys of the kept
 *     earlier blocks plus the keys c(t) * block_size .. t of its own block; the
 *     per-block partial results are merged by log-sum-exp.
 *
 * Conventions for every entry point:
 *   - q, out: bf16 [B, N, Hq, d]; k, v: bf16 [B, N, Hkv, d]; all contiguous.
 *     Query head h uses kv head floor(h / (Hq / Hkv)) (grouped-query sharing).
 *   - lse: fp32 [B, Hq, N], natural log of the softmax denominator of the
 *     scaled logits q.k / sqrt(d).
 *   - idx: int32 [B, Hq, N, topk], the kept blocks of each query in ascending
 *     order (so the own block c(t) comes last), padded with -1 when fewer than
 *     topk blocks exist.
 *   - All pointers are DEVICE pointers owned by the caller, 16-byte aligned.
 *     The library never frees or keeps them after the call returns.
 *   - Work is enqueued on `stream` (a cudaStream_t; 0 = legacy default stream)
 *     and runs asynchronously; an entry point returns once its work is queued.
 *   - Arguments are validated on the host before anything is queued; an invalid
 *     call returns a status code and queues nothing.
 *   - Asynchronous failures (a kernel wait that hit its limit, a launch error)
 *     are reported by moba_sync_status().
 *   - Supported: d = 128, Hq % Hkv == 0, 1 <= topk <= 64, block_size >= 1,
 *     1 <= N, B * N < 2^31, ceil(N / block_size) <= 16384, B and Hq <= 65535, and a
 *     device of compute capability 10.0 (sm_100a).
 */
#ifndef MOBA_H
#define MOBA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t, declared here so the header needs no CUDA include. */
typedef struct CUstream_st* moba_stream_t;

typedef enum {
    MOBA_OK = 0,
    MOBA_ERR_NULL = 1,           /* a required pointer is NULL */
    MOBA_ERR_SHAPE = 2,          /* unsupported sizes (see the list above) */
    MOBA_ERR_ALIGN = 3,          /* a pointer is not 16-byte aligned */
    MOBA_ERR_UNSUPPORTED = 4,    /* the current device is not sm_100 */
    MOBA_ERR_CUDA = 5,           /* a CUDA runtime call or launch failed */
    MOBA_ERR_OOM = 6,            /* the internal workspace could not be allocated */
    MOBA_ERR_DEVICE_TIMEOUT = 7, /* a kernel gave up waiting (bounded wait hit its limit) */
    MOBA_ERR_WORKSPACE = 8,      /* the caller's workspace is NULL or too small */
    MOBA_ERR_SELECTION = 9,      /* an injected selection is malformed (found on the device) */
    MOBA_ERR_VALUE = 10          /* an argument's values are invalid (found on the device): pooling weights */
} moba_status;

/* How a key block is summarised for the gate ("KIMI MoBA" blog: section 3 field
 * score_pooling = mean; section 6 suggests max or weighted pooling instead). */
typedef enum {
    MOBA_POOL_MEAN = 0,     /* mean of the block's keys (the method's default) */
    MOBA_POOL_MAX = 1,      /* feature-wise maximum over the block's keys */
    MOBA_POOL_WEIGHTED = 2  /* sum_p w[p] K[jB + p] / sum_p w[p], one weight per position in a block */
} moba_pooling;

/* Options of the extended entry points (moba_forward_ex, moba_gate_ex). Zero-initialise,
 * set struct_size = sizeof(moba_options), then the fields wanted; a NULL options pointer means
 * all defaults (mean pooling, MoBA attention). */
typedef struct moba_options {
    uint32_t struct_size;       /* sizeof(moba_options) */
    int32_t pooling;            /* moba_pooling */
    const float* pool_weights;  /* MOBA_POOL_WEIGHTED: DEVICE fp32 [block_size], every w >= 0 with a
                                   positive sum (checked on the device: MOBA_ERR_VALUE); else NULL */
    int32_t full_attention;     /* hybrid-layer switch ("KIMI MoBA" blog, section 3, hybrid_layers):
                                   1 = this layer uses full causal attention (no gating); 0 = MoBA */
    int32_t reserved;           /* must be 0 */
} moba_options;

/* Human-readable name of a status code (static string, never NULL). */
const char* moba_status_string(int status);

/*
 * Bytes of device workspace moba_forward_ws() needs for these sizes
 * (block mean keys, selection, per-block query lists and per-slot partial
 * outputs). Writes the count to *bytes. No device work.
 */
int moba_workspace_size(int B, int Hq, int Hkv, int64_t N, int d, int block_size, int topk,
                        size_t* bytes);

/*
 * The whole causal prefill forward: pooling, gating, top-k with the forced own
 * block, selection inversion, block-sparse attention and log-sum-exp merge.
 * Defined by: "MoBA project hub" page, Steps 1-3 (partition, parameter-less
 * gating, attention over the kept blocks merged by log-sum-exp); "MoBA
 * tech-report summary" page, section 2 (block partition, score s_i and top-k,
 * causality: no future block, own block always kept and masked causally);
 * "NSA vs MoBA" blog, section 1 (softmax(q k^T / sqrt(d)) v).
 * Writes out and lse. Allocates its workspace with cudaMallocAsync on `stream`
 * and frees it on the same stream.
 */
int moba_forward(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq,
                 int Hkv, int64_t N, int d, int block_size, int topk, moba_stream_t stream);

/* moba_forward with a caller-owned device workspace of at least moba_workspace_size() bytes
 * (256-byte aligned). The workspace must not be used by other work until the call's
 * stream work has finished. */
int moba_forward_ws(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq,
                    int Hkv, int64_t N, int d, int block_size, int topk, void* workspace,
                    size_t workspace_bytes, moba_stream_t stream);

/*
 * moba_forward_ws with options: the gate's pooling (mean, max, weighted) and the hybrid-layer
 * switch (full_attention = 1 runs dense causal attention, as moba_dense_causal, and needs no
 * workspace). A NULL workspace is allocated with cudaMallocAsync on `stream`, as moba_forward
 * does. Same layouts, ownership and errors as moba_forward_ws;
 * MOBA_ERR_SHAPE for an unknown pooling, a NULL pool_weights with MOBA_POOL_WEIGHTED, a
 * struct_size below sizeof(moba_options) or reserved != 0.
 */
int moba_forward_ex(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq,
                    int Hkv, int64_t N, int d, int block_size, int topk, const moba_options* options,
                    void* workspace, size_t workspace_bytes, moba_stream_t stream);

/*
 * Gating only: block mean pooling, scores <q_t, Kbar_j> over earlier blocks,
 * forced own block and top-k. Writes idx (int32 [B, Hq, N, topk]).
 * Defined by: "MoBA project hub" page, Step 2 (score of a block = inner product
 * of the query with the block's mean-pooled keys, no gate parameters, top-k);
 * "KIMI MoBA" blog, section 3 (score_pooling = mean, causal_mask,
 * current_block_force); "MoBA tech-report summary" page, section 2 (score s_i,
 * top-k, causality). Ties at the boundary go to the lower block index.
 * Allocates its small scratch (the block means) with cudaMallocAsync on `stream`.
 */
int moba_gate(const void* q, const void* k, int32_t* idx, int B, int Hq, int Hkv, int64_t N, int d,
              int block_size, int topk, moba_stream_t stream);

/* moba_gate with options (the pooling; full_attention must be 0). Allocates its scratch with
 * cudaMallocAsync on `stream`. */
int moba_gate_ex(const void* q, const void* k, int32_t* idx, int B, int Hq, int Hkv, int64_t N, int d,
                 int block_size, int topk, const moba_options* options, moba_stream_t stream);

/*
 * Attention with a given selection idx (same layout as moba_gate's output):
 * selection inversion, block-sparse attention and merge. Defined by: "MoBA
 * project hub" page, Step 3 (attention over the selected blocks, the own block
 * masked causally, partial results fused by log-sum-exp); "MoBA tech-report
 * summary" page, section 2, implementation steps 1-5 (queries grouped per key
 * block, attention per block, outputs combined by online softmax). Each row must list
 * distinct blocks <= c(t) and include c(t); a malformed row is skipped and
 * reported as MOBA_ERR_SELECTION by moba_sync_status(). Allocates its
 * workspace with cudaMallocAsync on `stream`.
 */
int moba_forward_selected(const void* q, const void* k, const void* v, const int32_t* idx, void* out,
                          float* lse, int B, int Hq, int Hkv, int64_t N, int d, int block_size,
                          int topk, moba_stream_t stream);

/* moba_forward_selected with a caller-owned workspace of at least moba_workspace_size() bytes. */
int moba_forward_selected_ws(const void* q, const void* k, const void* v, const int32_t* idx,
                             void* out, float* lse, int B, int Hq, int Hkv, int64_t N, int d,
                             int block_size, int topk, void* workspace, size_t workspace_bytes,
                             moba_stream_t stream);

/*
 * Dense causal softmax attention of the same shape (every key u <= t), the
 * comparison point of the method's speedup figures ("MoBA tech-report summary",
 * section 3). Writes out and lse. Needs no workspace.
 */
int moba_dense_causal(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq,
                      int Hkv, int64_t N, int d, moba_stream_t stream);

/*
 * Waits for `stream`, then returns and clears the library's device-side error
 * flag on the current device (MOBA_OK if no kernel reported a failure), or
 * MOBA_ERR_CUDA if the stream reported a CUDA error.
 */
int moba_sync_status(moba_stream_t stream);

/*
 * Failure-detection self-test. Launches one warp on `stream` that waits, through the
 * same bounded-wait routine the attention kernel uses, on an mbarrier that nothing
 * ever completes, with a wall-clock limit of limit_ns. The wait gives up after the
 * limit, records MOBA_ERR_DEVICE_TIMEOUT in the device error flag and the kernel
 * returns, so moba_sync_status(stream) then reports MOBA_ERR_DEVICE_TIMEOUT and the
 * context stays usable. Nothing faults, traps or hangs.
 * Returns MOBA_ERR_SHAPE for limit_ns outside [1e3, 1e10], MOBA_ERR_UNSUPPORTED /
 * MOBA_ERR_CUDA without a usable sm_100 device, MOBA_ERR_CUDA if the launch failed.
 */
int moba_selftest_wait_timeout(int64_t limit_ns, moba_stream_t stream);

/*
 * Stage timing for measurement. While enabled, every moba_forward* call records
 * CUDA events on its stream between its stages (0 pool, 1 gate, 2 selection
 * inversion, 3 attention, 4 merge; the first two are empty when the selection is
 * given). Returns the previous setting.
 */
int moba_stage_timing(int enable);

/*
 * Waits for the recorded calls, writes the milliseconds of each stage summed over
 * them into ms[0..n) (n <= 5 used), the number of calls into *calls (may be NULL),
 * and forgets the records.
 */
int moba_stage_times(float* ms, int n, int* calls);

/*
 * ---------------------------------------------------------------- backward
 * Gradients of sum(dout * out) for the causal prefill forward, with its selection held fixed:
 * the top-k choice is discrete, so gradients flow only through the attention over the kept keys
 * and the block summaries receive none ("MoBA tech-report summary" page, section 3, trains and
 * continues pre-training models with MoBA; the attention is softmax(q k^T / sqrt(d)) v as in the
 * "NSA vs MoBA" blog, section 1).
 *   dq = sum_u dS_tu k_u / sqrt(d), dk = sum_t dS_tu q_t / sqrt(d), dv = sum_t P_tu dout_t,
 *   P_tu = exp(q_t.k_u / sqrt(d) - lse_t), dS_tu = P_tu (dout_t.v_u - <dout_t, out_t>).
 * Inputs: q, k, v, out (the forward's output) and dout in the forward's layouts, lse fp32
 * [B, Hq, N] (the forward's); idx: the forward's selection (int32 [B, Hq, N, topk], as moba_gate
 * writes it) or NULL to run the gate again (same result). Outputs dq [B, N, Hq, d], dk, dv
 * [B, N, Hkv, d], bf16. A NULL workspace is allocated with cudaMallocAsync on `stream`;
 * otherwise at least moba_backward_workspace_size() bytes, 256-byte aligned.
 */
int moba_backward_workspace_size(int B, int Hq, int Hkv, int64_t N, int d, int block_size, int topk,
                                 size_t* bytes);

int moba_backward(const void* q, const void* k, const void* v, const void* out, const float* lse,
                  const void* dout, const int32_t* idx, void* dq, void* dk, void* dv, int B, int Hq, int Hkv,
                  int64_t N, int d, int block_size, int topk, void* workspace, size_t workspace_bytes,
                  moba_stream_t stream);

/*
 * ---------------------------------------------------------------- packed (varlen) batches
 * Sequences of different lengths packed back to back, as in the pages' FlashAttention pipeline
 * ("MoBA tech-report summary" page, section 2, implementation steps 1-5, a variable-length
 * kernel): sequence s holds tokens cu_seqlens[s] .. cu_seqlens[s+1] - 1 and is its own context
 * (its blocks start at its first token; no query attends another sequence's keys).
 * Layouts: q, out bf16 [total, Hq, d]; k, v bf16 [total, Hkv, d]; lse fp32 [Hq, total];
 * idx int32 [Hq, total, topk] (as moba_gate's rows). cu_seqlens is a HOST int64 array of
 * nseq + 1 non-decreasing offsets starting at 0 (empty sequences allowed), total =
 * cu_seqlens[nseq] < 2^31. Consecutive sequences of equal length run as one batch; others run
 * one after another on `stream`. A NULL workspace is allocated with cudaMallocAsync on
 * `stream`; otherwise at least moba_varlen_workspace_size() bytes, 256-byte aligned.
 */
int moba_varlen_workspace_size(const int64_t* cu_seqlens, int nseq, int Hq, int Hkv, int d, int block_size,
                               int topk, size_t* bytes);

/* The causal prefill forward of every packed sequence (options as in moba_forward_ex). */
int moba_forward_varlen(const void* q, const void* k, const void* v, void* out, float* lse,
                        const int64_t* cu_seqlens, int nseq, int Hq, int Hkv, int d, int block_size, int topk,
                        const moba_options* options, void* workspace, size_t workspace_bytes,
                        moba_stream_t stream);

/* The gate of every packed sequence (options as in moba_gate_ex). */
int moba_gate_varlen(const void* q, const void* k, int32_t* idx, const int64_t* cu_seqlens, int nseq, int Hq,
                     int Hkv, int d, int block_size, int topk, const moba_options* options, void* workspace,
                     size_t workspace_bytes, moba_stream_t stream);

/*
 * ---------------------------------------------------------------- decode step
 * One new query per sequence against its KV cache, with the prefill's gate: the query is the
 * token at position L - 1, scores the earlier full blocks j < c = floor((L - 1) / block_size) as
 * <q, Kbar_j>, keeps its own block c and the topk - 1 best earlier ones, and attends their keys
 * (the own block up to L - 1). Definition: "MoBA project hub" page, Steps 2-3, and "MoBA
 * tech-report summary" page, section 2, at the last row of the prefill. full_attention = 1 keeps
 * every block (a full-attention layer of a hybrid model; "KIMI MoBA" blog, section 3,
 * hybrid_layers: the pages decode with full attention).
 *
 * Layouts: q, out bf16 [B, Hq, d]; k, v bf16 [B, Lmax, Hkv, d] (a cache with room for Lmax tokens
 * per sequence, the first L filled; every sequence of the batch has length L); lse fp32 [B, Hq];
 * kbar fp64 [B, Hkv, kbar_rows, d], the block summaries written by moba_pool_cache; idx (optional,
 * may be NULL; not written with full_attention) int32 [B, Hq, topk], the kept blocks ascending,
 * own block last, -1 padded. Supported: Hq / Hkv <= 16, plus the limits above.
 */

/* Bytes of device workspace moba_decode needs. No device work. */
int moba_decode_workspace_size(int B, int Hq, int Hkv, int64_t L, int d, int block_size, int topk,
                               int full_attention, size_t* bytes);

/*
 * Block summaries of a KV cache for the gate of moba_decode: pools the full blocks
 * first_block .. floor(L / block_size) - 1 of k (bf16 [B, Lmax, Hkv, d]) into rows of kbar
 * (fp64 [B, Hkv, kbar_rows, d], kbar_rows >= floor(L / block_size)) with the options' pooling
 * (NULL: mean). A decoder that appends tokens pools each block once, when it becomes full.
 */
int moba_pool_cache(const void* k, double* kbar, int B, int Hkv, int64_t L, int64_t Lmax, int d,
                    int block_size, int64_t kbar_rows, int64_t first_block, const moba_options* options,
                    moba_stream_t stream);

/*
 * The decode step. kbar must hold the summaries of blocks 0 .. c - 1 (kbar_rows >= c; not read
 * with full_attention, may then be NULL). A NULL workspace is allocated with cudaMallocAsync on
 * `stream`; otherwise at least moba_decode_workspace_size() bytes, 256-byte aligned.
 */
int moba_decode(const void* q, const void* k, const void* v, const double* kbar, int64_t kbar_rows, void* out,
                float* lse, int32_t* idx, int B, int Hq, int Hkv, int64_t L, int64_t Lmax, int d, int block_size,
                int topk, int full_attention, void* workspace, size_t workspace_bytes, moba_stream_t stream);

/*
 * moba_gate without any device allocation, for callers that cannot allocate
 * while they run (serving engines that pre-plan every byte of HBM for their KV
 * cache, embedders with a fixed memory budget). The MoBA pages have no
 * counterpart: this is a library convenience. Same arguments and results as
 * moba_gate. It always runs the fp64 CUDA-core gate (whose only scratch is the
 * block means), so its selections are moba_gate's, but at long sequences it is
 * slower than moba_gate's default tensor-core gate. Its scratch is a fixed
 * 8 MiB device array inside the library, held by every GPU that loads it until exit.
 *   - Limit: B * Hkv * floor(N / block_size) <= 8192, else MOBA_ERR_SHAPE.
 *   - The first call on a device looks up the array's device address with that
 *     device current; make that first call before any stream capture. The
 *     address is looked up again when the current CUDA context changed since
 *     (for example after a device reset).
 *   - All calls share the array: calls that overlap on the GPU race on it.
 *     Nothing in it needs clearing (each call overwrites what it reads).
 */
int moba_gate_noalloc(const void* q, const void* k, int32_t* idx, int B, int Hq, int Hkv, int64_t N, int d,
                      int block_size, int topk, moba_stream_t stream);

/* Text of the last CUDA runtime error the library met on the calling host thread
 * (for messages after MOBA_ERR_CUDA); "no error" if there was none. Static string. */
const char* moba_last_error_string(void);

/* Number of kernels the library has launched in this process (all devices). */
uint64_t moba_launch_count(void);

/* TEST HOOK, process-wide. Implementation of the attention step used by every later call
 * from any thread of the process: 0 = tensor-core kernel (default), 1 = the simple
 * CUDA-core kernel kept only as an independent cross-check in the tests. Values other
 * than 0 and 1 are refused (MOBA_ERR_SHAPE is returned and nothing changes); otherwise
 * returns the previous value. The switch is atomic, but calls that run while another
 * thread changes it may use either kernel: set it once, before any concurrent use. */
int moba_set_attention_impl(int impl);

/* TEST HOOK, process-wide, same rules as moba_set_attention_impl: the gate used by every
 * later call, 0 = default (tensor-core gate with exact fp64 boundary re-scoring), 1 = the
 * CUDA-core fp64 gate kept as a cross-check. Returns the previous value, or MOBA_ERR_SHAPE
 * for any other value. */
int moba_set_gate_impl(int impl);

#ifdef __cplusplus
}
#endif

#endif /* MOBA_H */
