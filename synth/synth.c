/*
 * Seeded synthetic inputs for the MoBA causal prefill forward.
 *
 * This module only draws numbers. It holds none of the attention method's
 * arithmetic and is shared by the CPU oracle tests and the GPU harness so that
 * both see identical bytes.
 *
 * Generator (counter based, so any element can be drawn on its own):
 *   - splitmix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
 *     generators", OOPSLA 2014): output i of a stream with seed `key` is the
 *     splitmix64 finaliser applied to key + (i + 1) * 0x9E3779B97F4A7C15.
 *   - uniform: the top 53 bits of an output, scaled by 2^-53.
 *   - normal: the Box-Muller transform (Box & Muller 1958) on the output pair
 *     (2p, 2p + 1); element 2p takes the cosine branch, 2p + 1 the sine branch.
 *   - every value is formed in double precision and rounded once to bfloat16
 *     with round-to-nearest-even.
 *
 * Workload recipe (the value distribution the MoBA pages' configurations use):
 *   Q, V ~ N(0, 1); K = N(0, 1) + c[b, h, j] * 1_d with c ~ N(0, 0.5^2) drawn
 *   once per (batch, kv head, key block j = floor(t / block_size)).
 * Layout: bf16 [B, N, H, d] contiguous.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

enum { SYNTH_Q = 1, SYNTH_K = 2, SYNTH_V = 3, SYNTH_KOFF = 4 };

static inline uint64_t sm64_fin(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

static inline uint64_t sm64_at(uint64_t key, uint64_t i) {
    return sm64_fin(key + (i + 1ull) * 0x9E3779B97F4A7C15ull);
}

/* Stream key for (seed, tensor id): one splitmix64 step keyed by both. */
uint64_t synth_stream_key(uint64_t seed, uint32_t tensor_id) {
    return sm64_fin(seed * 0x100000001B3ull + (uint64_t)tensor_id * 0xD6E8FEB86659FD93ull);
}

static inline double u53(uint64_t z) { return (double)(z >> 11) * 0x1.0p-53; }

/* Standard normal number `i` of the stream `key`. */
double synth_normal_at(uint64_t key, uint64_t i) {
    uint64_t p = i >> 1;
    double u1 = ((double)(sm64_at(key, 2 * p) >> 11) + 1.0) * 0x1.0p-53; /* (0, 1] */
    double u2 = u53(sm64_at(key, 2 * p + 1));                            /* [0, 1) */
    double r = sqrt(-2.0 * log(u1));
    double th = 6.283185307179586476925286766559 * u2;
    return (i & 1) ? r * sin(th) : r * cos(th);
}

/* Round a double to bfloat16 (round to nearest, ties to even), returning the
 * 16-bit pattern. Values are far inside the bf16 exponent range here, so the
 * rounding is done on the double's significand and the result is exact in
 * float before its top half is taken. */
uint16_t synth_bf16_rne(double x) {
    uint64_t b;
    memcpy(&b, &x, 8);
    if (((b >> 52) & 0x7FF) == 0x7FF) { /* inf / nan: not produced by this module */
        float f = (float)x;
        uint32_t u;
        memcpy(&u, &f, 4);
        return (uint16_t)(u >> 16);
    }
    const uint64_t drop = 45; /* 52 - 7 explicit bf16 fraction bits */
    uint64_t bias = ((1ull << (drop - 1)) - 1ull) + ((b >> drop) & 1ull);
    b += bias;
    b &= ~((1ull << drop) - 1ull);
    double y;
    memcpy(&y, &b, 8);
    float f = (float)y;
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}

/* Fill a bf16 tensor [B, N, H, d] with N(0,1) numbers from (seed, tensor_id). */
void synth_fill_normal(uint16_t* out, uint64_t seed, uint32_t tensor_id, int64_t count) {
    uint64_t key = synth_stream_key(seed, tensor_id);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; ++i) out[i] = synth_bf16_rne(synth_normal_at(key, (uint64_t)i));
}

/* Per-block key offset c[b, h, j] (before rounding), j < nblk = ceil(N / block_size). */
double synth_key_offset(uint64_t seed, int64_t b, int64_t h, int64_t j, int64_t Hkv, int64_t nblk) {
    uint64_t key = synth_stream_key(seed, SYNTH_KOFF);
    return 0.5 * synth_normal_at(key, (uint64_t)((b * Hkv + h) * nblk + j));
}

/* K[b, t, h, :] = N(0,1) + c[b, h, floor(t / block_size)], rounded once to bf16. */
void synth_fill_keys(uint16_t* out, uint64_t seed, int64_t B, int64_t N, int64_t Hkv, int64_t d,
                     int64_t block_size) {
    uint64_t key = synth_stream_key(seed, SYNTH_K);
    int64_t nblk = (N + block_size - 1) / block_size;
#pragma omp parallel for schedule(static)
    for (int64_t row = 0; row < B * N * Hkv; ++row) {
        int64_t h = row % Hkv;
        int64_t t = (row / Hkv) % N;
        int64_t b = row / (Hkv * N);
        double c = synth_key_offset(seed, b, h, t / block_size, Hkv, nblk);
        for (int64_t e = 0; e < d; ++e) {
            int64_t i = row * d + e;
            out[i] = synth_bf16_rne(synth_normal_at(key, (uint64_t)i) + c);
        }
    }
}

/* Heads [h0, h1) of the N(0,1) tensor [B, N, H, d] of stream (seed, tensor_id), written as
 * [B, N, h1 - h0, d]: element (b, t, h, e) is number ((b * N + t) * H + h) * d + e of the
 * stream, the same value the whole tensor holds there. */
void synth_fill_normal_heads(uint16_t* out, uint64_t seed, uint32_t tensor_id, int64_t B, int64_t N,
                             int64_t H, int64_t d, int64_t h0, int64_t h1) {
    uint64_t key = synth_stream_key(seed, tensor_id);
    int64_t nh = h1 - h0;
#pragma omp parallel for schedule(static)
    for (int64_t row = 0; row < B * N * nh; ++row) {
        int64_t h = h0 + row % nh;
        int64_t bt = row / nh;
        for (int64_t e = 0; e < d; ++e)
            out[row * d + e] = synth_bf16_rne(synth_normal_at(key, (uint64_t)((bt * H + h) * d + e)));
    }
}

/* Heads [h0, h1) of the key tensor of synth_fill_keys, written as [B, N, h1 - h0, d]. */
void synth_fill_keys_heads(uint16_t* out, uint64_t seed, int64_t B, int64_t N, int64_t Hkv, int64_t d,
                           int64_t block_size, int64_t h0, int64_t h1) {
    uint64_t key = synth_stream_key(seed, SYNTH_K);
    int64_t nblk = (N + block_size - 1) / block_size;
    int64_t nh = h1 - h0;
#pragma omp parallel for schedule(static)
    for (int64_t row = 0; row < B * N * nh; ++row) {
        int64_t h = h0 + row % nh;
        int64_t t = (row / nh) % N;
        int64_t b = row / (nh * N);
        double c = synth_key_offset(seed, b, h, t / block_size, Hkv, nblk);
        int64_t grow = (b * N + t) * Hkv + h;
        for (int64_t e = 0; e < d; ++e)
            out[row * d + e] = synth_bf16_rne(synth_normal_at(key, (uint64_t)(grow * d + e)) + c);
    }
}
