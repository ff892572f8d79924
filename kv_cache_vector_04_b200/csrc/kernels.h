// Launch interfaces between the host API (api.cu) and the kernels.
#pragma once
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace tq {

struct DevTables;

// A cache format: head dim, key cell bits, value cell bits, QJL sketch on keys.
struct Format {
    int d, kb, vb, qjl;
};

struct QuantizeArgs {
    const __half* k;          // [B][Hkv][T][d]
    const __half* v;          // [B][Hkv][T][d]
    const int32_t* start_pos; // [B]
    uint8_t* cache;           // [B][Hkv][capacity/16][tile_bytes]
    int B, Hkv, T, capacity;
    long long tile_bytes;
};

// Geometry of one attention call.
struct AttendPlan {
    int groups;     // head groups of 8 per kv head: ceil((Hq/Hkv) / 8)
    int tiles;      // ceil(max_len / 16)
    int nsplit;     // tq_scores: splits of the context per (b, kv head, group)
    int tps;        // tq_scores: tiles per split
    int ctas;       // tq_attend: CTAs of the stream-K split kernel
    size_t qfrag_bytes, prefix_bytes, partial_bytes, total_bytes;
};

struct AttendArgs {
    const void* q;            // [B][Hq][d] fp16 / bf16
    int q_bf16;
    const int32_t* seq_len;   // [B]
    const uint8_t* cache;
    int B, Hq, Hkv, capacity, max_len;
    long long tile_bytes;
    uint32_t* qfrag;          // workspace: [B][Hkv*groups][d/16][64] uint4 query fragments (codebook fp16, QJL int8)
    long long* prefix;        // workspace: [B + 1] first flattened tile of each sequence's units
    float* partial;           // workspace: [ctas + B*Hkv*groups][8][d + 2], slot = CTA + unit
    float* out;               // [B][Hq][d] (attend) or scores [B][Hq][max_len]
    AttendPlan plan;
    // fused append (tq_append_attend with 1 <= T <= 16; k_new == nullptr otherwise)
    const __half* k_new;      // [B][Hkv][T][d]
    const __half* v_new;      // [B][Hkv][T][d]
    const int32_t* start_pos; // [B]
    int T;
    uint8_t* cache_w;         // the cache, writable
    // tq_attend_cudacore: 1 or 2 runs the CUDA-core split kernel (QJL term by
    // sign-nibble tables or by bit-plane popcounts) in place of the tensor-core one
    int cc_mode;
};

cudaError_t launch_quantize(const Format& f, const DevTables& tb, const QuantizeArgs& a,
                            cudaStream_t st);
cudaError_t launch_attend(const Format& f, const DevTables& tb, const AttendArgs& a,
                          bool scores, cudaStream_t st);
cudaError_t launch_copy(const void* src, void* dst, size_t bytes, cudaStream_t st);
cudaError_t launch_attend_d64(const Format& f, const DevTables& tb, const AttendArgs& a, bool scores,
                             cudaStream_t st);
cudaError_t launch_attend_d128(const Format& f, const DevTables& tb, const AttendArgs& a, bool scores,
                              cudaStream_t st);
cudaError_t launch_attend_d256(const Format& f, const DevTables& tb, const AttendArgs& a, bool scores,
                              cudaStream_t st);

AttendPlan plan_attend(const Format& f, int B, int Hq, int Hkv, int max_len, int num_sms);
// Split CTAs resident per SM for a format (its shared memory and registers).
int attend_ctas_per_sm(const Format& f);

// Every built format, for the launch tables: X(D, KB, VB, QJL).
#define TQ_FORMATS_D(X, D) \
    X(D, 1, 2, 1) X(D, 2, 3, 1) X(D, 3, 4, 1) X(D, 7, 4, 1) X(D, 2, 2, 0) X(D, 3, 3, 0) X(D, 4, 4, 0) \
    X(D, 3, 4, 0)
#define TQ_FORMATS(X) TQ_FORMATS_D(X, 64) TQ_FORMATS_D(X, 128) TQ_FORMATS_D(X, 256)

}  // namespace tq
