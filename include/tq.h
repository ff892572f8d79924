/*
 * tq.h — C ABI of the TurboQuant KV-cache library for NVIDIA B200 (sm_100a).
 *
 * TurboQuant compresses each key and value vector of an LLM KV cache, per
 * token and per head, in three steps ("[Benchmark] TurboQuant 實測：KV Cache
 * 3-bit 壓縮，真的零損失？", ai-muninn.com, §"TurboQuant 是什麼：30 秒懶人包";
 * "turboquant-kvquant-vllm-benchmark", ai-coding.wiselychen.com,
 * §"TurboQuant 是什麼"):
 *   1. a random rotation Pi = H D / sqrt(d) of the unit vector u = x / |x|
 *      (a random ±1 diagonal D, then the Walsh–Hadamard transform H);
 *   2. an optimal Lloyd–Max scalar quantizer per rotated coordinate, with no
 *      calibration data (keys: b-1 bits; values: b bits);
 *   3. for keys only, a 1-bit QJL sketch of the residual r = y - c[idx]:
 *      the signs of S r for an m x d Gaussian S (m = d), with |r| stored.
 * Attention logits are then estimated without bias as
 *   l_n = |k_n| (<Pi q, c[idx_n]> + |r_n| sqrt(pi/2)/m <S Pi q, signs_n>) / sqrt(d),
 * and values are accumulated in the rotated domain with one inverse rotation
 * per output.
 *
 * Conventions for every call:
 *  - Return 0 (TQ_OK) on success, a negative TQ_ERR_* code otherwise; nothing
 *    is launched when an argument check fails.
 *  - Pointers marked "device" are device pointers on the device that was
 *    current at tq_init; "host" pointers are host memory. The caller owns all
 *    buffers; the library never frees caller memory and (except in tq_init)
 *    never allocates device memory.
 *  - Kernels launch asynchronously on the caller's `stream` (a cudaStream_t
 *    passed as void*; NULL = the legacy default stream). Only tq_init,
 *    tq_destroy and tq_status synchronize.
 *  - Conditions that depend on device-side values (a start position or a
 *    sequence length out of range, a norm that saturates fp16) never trap:
 *    the kernel skips the affected write or clamps, and sets a bit in a sticky
 *    status word read by tq_status.
 *  - Calls on one context may run concurrently only if they touch disjoint
 *    cache regions and workspaces.
 */
#ifndef TQ_H
#define TQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---------------------------------------------------------------- codes */
#define TQ_OK 0
#define TQ_ERR_INVALID_ARG (-1) /* a NULL pointer, a size out of range, ...  */
#define TQ_ERR_UNSUPPORTED (-2) /* d or bits outside the supported set       */
#define TQ_ERR_CUDA (-3)        /* a CUDA runtime call or a launch failed     */
#define TQ_ERR_WORKSPACE (-4)   /* the workspace is smaller than required     */
#define TQ_ERR_DEVICE (-5)      /* called with another device current         */

/* sticky device status bits (tq_status) */
#define TQ_STATUS_CAPACITY 0x1u  /* tq_quantize: start_pos < 0 or start_pos+T > capacity; batch item skipped */
#define TQ_STATUS_SEQ_LEN 0x2u   /* tq_attend/tq_scores: seq_len < 0 or > min(max_len, capacity); clamped */
#define TQ_STATUS_NORM_SAT 0x4u  /* tq_quantize: a norm exceeded 65504 and was stored as 65504 */
#define TQ_STATUS_WAIT_TIMEOUT 0x8u /* tq_attend: a copy into shared memory did not complete within the
                                     * kernel's bounded wait; that call's output is unspecified */

#define TQ_TILE 16 /* tokens per packed tile */

/* dtypes of query input */
#define TQ_CODEBOOK_GAUSS 0 /* Lloyd–Max for N(0, 1/d), the pages' coordinate model */
#define TQ_CODEBOOK_BETA 1  /* Lloyd–Max for the exact marginal: (1 + y)/2 ~ Beta((d-1)/2, (d-1)/2) */

#define TQ_DTYPE_F16 0
#define TQ_DTYPE_BF16 1

typedef struct tq_ctx tq_ctx; /* opaque: the codebook, rotation and QJL tables of one (d, bits, seed) */

/* Sizes of the packed cache (see "Packed cache format" below). */
typedef struct {
    int32_t d;                 /* head dimension: 64, 128 or 256                          */
    int32_t bits;              /* b = B_V (TurboQuant at b bits: K b-1 + 1 QJL; V b)      */
    int32_t m;                 /* QJL rows, = d                                           */
    int32_t kbits, vbits;      /* B_K, B_V: key and value cell bits                       */
    int32_t tile;              /* TQ_TILE                                                 */
    int64_t k_bytes_per_token; /* (B_K+qjl)*d/8 + 2 + 2*qjl: codes, signs, |k|, rho       */
    int64_t v_bytes_per_token; /* B_V*d/8 + 2: codes + fp16 |v|                           */
    int64_t tile_bytes;        /* TQ_TILE * (k_bytes_per_token + v_bytes_per_token)       */
    int64_t code_bytes;        /* 2*W*d, W = B_K + qjl + B_V: the tile's code region      */
    int32_t chunk_bytes;       /* 16, 8 or 4: the largest dividing a lane string (W*d/16)  */
    int32_t qjl;               /* 1: keys carry the QJL sketch and rho; 0: MSE-only keys  */
} tq_layout;

/* A packed cache of B sequences x Hkv kv heads x `capacity` token slots.
 * data: device, B*Hkv*(capacity/16)*tile_bytes bytes, 16-byte aligned, laid
 * out [B][Hkv][capacity/16 tiles][tile_bytes]. capacity is a positive
 * multiple of TQ_TILE. Slots that were never written hold whatever the caller
 * put there; they are never read for positions >= the sequence length. */
typedef struct {
    void* data;
    int32_t B, Hkv, capacity;
} tq_cache;

/*
 * Packed cache format (one 16-token tile of one (batch, kv head)). A format is
 * (B_K, B_V, qjl); TurboQuant at b bits is (b-1, b, 1), where W = B_K + qjl +
 * B_V = 2b, so that the code region is 4bd bytes and a lane string b*d/8 bytes:
 *  bytes [0, 2Wd): the code region. It holds 32 "lane strings" of W*d/16 bytes,
 *    stored in chunks of chunk_bytes: chunk c of lane l is at byte
 *    (c*32 + l)*chunk_bytes; a lane string is its chunks in order and bit k of
 *    it is bit k%8 of its byte k/8. Lane l = 4g + t (g < 8, t < 4) holds, for
 *    p = 4kk + r (kk < d/16, r < 4) and e in {0, 1}:
 *      K code of token g + 8(r&1), coordinate 16kk + 8(r>>1) + 2t + e:
 *        B_K bits at 2*B_K*p + e*B_K;
 *      (qjl = 1) QJL sign bit of the same token, row 16kk + 8(r>>1) + 2t + e:
 *        at B_K*d/2 + 32*(p/16) + 16e + (p%16)  (1 = S r >= 0);
 *      V code of token 2t + 8(r>>1) + e, coordinate 16kk + g + 8(r&1):
 *        B_V bits at (B_K+qjl)*d/2 + 2*B_V*p + e*B_V.
 *    Format (3, 4, 1) (TurboQuant at 4 bits) instead keeps each key pair and
 *    two sign bits in one byte: the K code at 8p + 3e (bits 0..5 of byte p),
 *    the sign at 32*(p/4) + 16e + a, a = 6, 7, 14, 15 for p%4 = 0, 1, 2, 3
 *    (bits 6 and 7 of the bytes of word p/4); its V codes as above.
 *    Format (2, 3, 1) (TurboQuant at 3 bits) keeps each value pair and two
 *    sign bits in one byte instead: the K codes as above (the first B_K*d/2
 *    bits), then the V code at B_K*d/2 + 8p + 3e (bits 0..5 of byte p of that
 *    region) and the sign at B_K*d/2 + 32*(p/4) + 16e + a, a as above. With
 *    4-bit value cells every V pair is one byte, and with (4, 4, 0) every K
 *    pair too: the decoder turns such a byte into its table row with one
 *    byte permute.
 *    (Lane l's bits are exactly the operands that lane l of a warp needs for
 *    the m16n8k16 tensor-core fragments of the attention kernel, so each lane
 *    streams its own bytes with 128-bit coalesced loads.)
 *  then the K norms: qjl = 1: 64 bytes, for g = 0..7, fp16 {|k_g|, rho_g,
 *    |k_g+8|, rho_g+8}; qjl = 0: 32 bytes, fp16 {|k_g|, |k_g+8|};
 *  then the V norms: 32 bytes; for g = 0..7, fp16 {|v_g|, |v_g+8|}.
 * Codes are cell indices of the sorted codebook (0 = most negative). Norms are
 * fp16, round to nearest even, saturating at 65504.
 */

/* Build the tables for head dimension d in {64, 128, 256}, b = bits in
 * {2, 3, 4} and a 64-bit seed, on the current device:
 *  - Lloyd–Max codebooks for N(0, 1/d) with 2^(b-1) levels (keys) and 2^b
 *    levels (values): fp64 Lloyd iteration, symmetric, rounded once to fp32;
 *    boundaries are the fp32 midpoints ("Lloyd-Max Codebook" section of the
 *    ai-muninn page; the Gaussian coordinate model of a rotated unit vector);
 *  - D: d signs, D_i = -1 iff the top bit of SplitMix64 draw i of stream 0 is set;
 *  - S: m x d, N(0,1) by Box–Muller from SplitMix64 stream 1, each entry
 *    rounded once to fp16.
 * Draw k of stream s is output k+1 of SplitMix64 started at
 * seed ^ (0x5851F42D4C957F2D * (s+1)).
 * *out receives a new context (owned by the caller; free with tq_destroy).
 * Allocates a small device block (under 1 MB: about 0.9 MB for 4-bit key pairs at
 * d = 256, about 120 KB for TurboQuant at 3 bits and d = 128) and synchronizes. */
int tq_init(int d, int bits, uint64_t seed, tq_ctx** out);

/* tq_init for any built format (B_K = kbits, B_V = vbits, QJL sketch on keys
 * iff qjl = 1); tq_init(d, b, ...) is tq_init_ex(d, b - 1, b, 1, ...). Built:
 * qjl = 1 with kbits = vbits - 1 and vbits in {2, 3, 4} (TurboQuant); qjl = 1
 * with (kbits, vbits) = (7, 4): the k8v4 variant of the table below, read as
 * TurboQuant keys at 8 bits (7-bit cells + the QJL sketch) with 4-bit values;
 * and the MSE-only key formats qjl = 0 with (kbits, vbits) in {(2,2), (3,3), (4,4),
 * (3,4)}: the "nc" and k3v4-nc variants of the method table in the vLLM
 * section ("vLLM 工程師的實測") of turboquant-kvquant-vllm-benchmark, read as
 * "no QJL correction" ([MUNINN] §"MSE-Only vs QJL" contrasts the two). Without
 * QJL the logit is |k| <Pi q, cK[idx]> / sqrt(d), the biased MSE-only
 * estimate. Other formats return TQ_ERR_UNSUPPORTED. */
int tq_init_ex(int d, int kbits, int vbits, int qjl, int codebook, uint64_t seed, tq_ctx** out);
/* codebook (tq_init_ex): TQ_CODEBOOK_GAUSS, or TQ_CODEBOOK_BETA for the exact
 * distribution of a rotated unit-vector coordinate, which the N(0, 1/d) model
 * approximates (turboquant-kvquant-vllm-benchmark, "TurboQuant 是什麼", step
 * 1: the rotation concentrates the coordinates as a Beta distribution). */

/* One codebook alone, on the host (no device, no context): B in 1..7 bits,
 * d >= 3; fp32 centroids[2^B] and boundaries[2^B - 1] (fp32 midpoints). */
int tq_build_codebook(int B, int d, int codebook, float* centroids, float* bounds);

/* Free a context and its device tables. NULL is ignored. */
void tq_destroy(tq_ctx* ctx);

/* Fill *out with the sizes of the packed format of this context. */
int tq_cache_layout(const tq_ctx* ctx, tq_layout* out);

/* Bytes of a cache of B x Hkv x capacity tokens (capacity a multiple of 16). */
int tq_cache_bytes(const tq_ctx* ctx, int B, int Hkv, int capacity, size_t* bytes);

/* Host copies of the tables, for checking (any pointer may be NULL):
 * centroids_k[2^B_K], bounds_k[2^B_K-1], centroids_v[2^B_V], bounds_v[2^B_V-1]
 * (fp32), signs[d] (int8 ±1), S[m*d] (fp32, row-major, fp16-exact values). */
int tq_get_tables(const tq_ctx* ctx, float* centroids_k, float* bounds_k, float* centroids_v,
                  float* bounds_v, int8_t* signs, float* S);

/* The same tables computed on the host only (no device needed, no context). */
int tq_build_tables(int d, int bits, uint64_t seed, float* centroids_k, float* bounds_k,
                    float* centroids_v, float* bounds_v, int8_t* signs, float* S);

/* Quantize and append T tokens per sequence (steps 1–3 above, then packing).
 *  k, v:       device, fp16, [B][Hkv][T][d] contiguous (16-byte aligned).
 *  start_pos:  device, int32[B]: token t of sequence b goes to slot
 *              start_pos[b] + t. If start_pos[b] < 0 or start_pos[b] + T >
 *              cache->capacity, nothing of sequence b is written and
 *              TQ_STATUS_CAPACITY is set.
 *  cache:      host struct describing the device cache; cache->B and
 *              cache->Hkv must equal B and Hkv.
 * Slots of a tile that are not written keep their previous bits. T = 0 is a
 * no-op. One launch; asynchronous on `stream`. */
int tq_quantize(tq_ctx* ctx, const void* k, const void* v, int B, int Hkv, int T,
                const int32_t* start_pos, const tq_cache* cache, void* stream);

/* Workspace bytes tq_attend / tq_scores need for (B, Hq, Hkv, max_len). */
int tq_attend_workspace(const tq_ctx* ctx, int B, int Hq, int Hkv, int max_len, size_t* bytes);

/* One decode-attention step over the packed cache (split-K flash decoding):
 *  q:        device, [B][Hq][d], fp16 or bf16 (q_dtype), contiguous.
 *  Hq:       a multiple of cache->Hkv; query head h reads kv head h / (Hq/Hkv).
 *  seq_len:  device, int32[B]: tokens [0, seq_len[b]) of sequence b are
 *            attended. Values outside [0, min(max_len, capacity)] are clamped
 *            and set TQ_STATUS_SEQ_LEN.
 *  max_len:  host upper bound of seq_len (sizes the split-K grid), 0..capacity.
 *  out:      device, fp32 [B][Hq][d]: softmax(l) weighted sum of the
 *            dequantized values (zero when seq_len[b] = 0).
 *  workspace: device scratch of at least tq_attend_workspace(...) bytes,
 *            256-byte aligned; its contents need no initialisation.
 * Three launches on `stream`: the query prologue (Pi q, S Pi q for each group
 * of 8 query heads), the split kernel, and the cross-split reduction with the
 * inverse rotation. */
int tq_attend(tq_ctx* ctx, const void* q, int q_dtype, int B, int Hq, const tq_cache* cache,
              const int32_t* seq_len, int max_len, float* out, void* workspace,
              size_t workspace_bytes, void* stream);

/* One decode step of a layer: append T new tokens to the cache, then attend.
 * The result is that of tq_quantize(ctx, k, v, B, Hkv, T, start_pos, cache,
 * stream) followed by tq_attend(ctx, q, q_dtype, B, Hq, cache, seq_len,
 * max_len, out, workspace, workspace_bytes, stream), with Hkv = cache->Hkv:
 *  k, v:      device, fp16 [B][Hkv][T][d], contiguous, 16-byte aligned.
 *  T:         new tokens per sequence, >= 0.
 *  start_pos: device, int32[B]: the new tokens go to positions
 *             [start_pos[b], start_pos[b] + T) (TQ_STATUS_CAPACITY as in
 *             tq_quantize). seq_len normally equals start_pos + T.
 * The other arguments are those of tq_attend. For 1 <= T <= 16 the new tokens
 * are quantized inside the first attention launch, by one CTA per (sequence,
 * kv head) working on shared-memory copies of the (at most two) tiles they
 * touch: three launches per call. For T > 16 the quantize kernel runs first.
 * This is the per-layer decode step the pages' generation-speed measurements
 * time ("[Benchmark] TurboQuant 實測：KV Cache 3-bit 壓縮，真的零損失？",
 * §"GB10 速度"). */
int tq_append_attend(tq_ctx* ctx, const void* q, int q_dtype, const void* k, const void* v, int B,
                     int Hq, int T, const int32_t* start_pos, const tq_cache* cache,
                     const int32_t* seq_len, int max_len, float* out, void* workspace,
                     size_t workspace_bytes, void* stream);

/* The estimated attention logits alone (the "inner product" of the pages'
 * speed test): scores[b][h][n] = l_n for n < seq_len[b], -inf for
 * seq_len[b] <= n < max_len. scores: device fp32 [B][Hq][max_len]. Same
 * arguments and workspace as tq_attend. */
int tq_scores(tq_ctx* ctx, const void* q, int q_dtype, int B, int Hq, const tq_cache* cache,
              const int32_t* seq_len, int max_len, float* scores, void* workspace,
              size_t workspace_bytes, void* stream);

/* tq_attend computed on CUDA cores instead of tensor cores, kept as a measured
 * comparison for the tensor-core split kernel (it is several times slower).
 * The operation, the arguments, the workspace and the prologue and reduce
 * launches are those of tq_attend; only the split kernel differs. It reads the
 * tiles with the same bulk copies and the same stream-K split, and writes the
 * same partials. Per unit of 8 query heads it builds shared-memory lookup tables:
 *  - the logits' codebook term sum_i q~_i c[idx_i] from a table of
 *    q~_i x c[code] per (coordinate, code, head);
 *  - the QJL term sum_j (2 s_j - 1) x_j (x = S q~ in the fixed point of the
 *    tensor-core path) from one of two tables:
 *    qjl_mode TQ_CC_QJL_NIBBLE: per group of 4 signs, the 16 signed sums;
 *    qjl_mode TQ_CC_QJL_POPCOUNT: the 16 bit planes of the fixed-point x,
 *    sum_b w_b popc(signs & plane_b).
 * P V runs as fp32 FMAs. Built for d = 128 with TurboQuant at 4 bits only
 * (tq_init(128, 4, ...)); any other context returns TQ_ERR_UNSUPPORTED, and
 * any other qjl_mode returns TQ_ERR_INVALID_ARG. The estimator is the one
 * tq_attend implements (the logit estimate at the top of this file, from
 * §"TurboQuant 是什麼：30 秒懶人包" of the ai-muninn page). */
#define TQ_CC_QJL_NIBBLE 1
#define TQ_CC_QJL_POPCOUNT 2
int tq_attend_cudacore(tq_ctx* ctx, const void* q, int q_dtype, int B, int Hq, const tq_cache* cache,
                       const int32_t* seq_len, int max_len, float* out, void* workspace,
                       size_t workspace_bytes, int qjl_mode, void* stream);

/* tq_attend without a workspace argument, for callers that cannot allocate
 * device memory: runtimes whose device memory belongs to an allocator they do
 * not control, and serving loops that forbid allocation after start-up. (The
 * pages describe no such call; it is an addition of this library.) The
 * scratch is a static device array of TQ_NOALLOC_SCRATCH_BYTES that exists on
 * every GPU that loads the library until the process exits; calls needing
 * more (tq_attend_workspace) return TQ_ERR_WORKSPACE without launching
 * anything. The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current and keeps it for the life
 * of the process; do not use the library across a cudaDeviceReset (which also invalidates every
 * context's device tables). All calls share the one array: calls that
 * overlap on a GPU race and must be serialized by the caller. No memory is
 * allocated or freed. Other arguments, results and launches are those of
 * tq_attend. */
#define TQ_NOALLOC_SCRATCH_BYTES (16u << 20)
int tq_attend_noalloc(tq_ctx* ctx, const void* q, int q_dtype, int B, int Hq, const tq_cache* cache,
                      const int32_t* seq_len, int max_len, float* out, void* stream);

/* Read and clear the sticky status bits of this context (synchronizes the
 * device). */
int tq_status(tq_ctx* ctx, uint32_t* flags);

/* Device-to-device copy kernel used to measure HBM bandwidth in the same
 * process (bytes a multiple of 16, both pointers 16-byte aligned). */
int tq_copy(const void* src, void* dst, size_t bytes, void* stream);

/* Static description of an error code. */
const char* tq_strerror(int code);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H */
