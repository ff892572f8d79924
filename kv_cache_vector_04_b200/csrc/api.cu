// Host side of the C ABI declared in include/tq.h: contexts, argument checks,
// device tables and kernel launches.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <algorithm>
#include <cstring>
#include <new>
#include <vector>

#include "device_common.cuh"
#include "kernels.h"
#include "tables.h"
#include "tq.h"

struct tq_ctx {
    int d = 0, bits = 0, kbits = 0, vbits = 0, qjl = 1, device = 0, num_sms = 148;
    tq::HostTables host;
    void* dev_block = nullptr;
    tq::DevTables tables{};
};

namespace {

// The built formats (B_K, B_V, qjl): TurboQuant at 2, 3, 4 bits; TurboQuant
// keys at 8 bits with 4-bit values ("k8v4": 7-bit cells + QJL); and the
// MSE-only key formats 2/2, 3/3, 4/4 and 3/4 bits.
bool supported(int d, int kbits, int vbits, int qjl)
{
    if (d != 64 && d != 128 && d != 256) return false;
    if (qjl == 1)
        return (vbits >= 2 && vbits <= 4 && kbits == vbits - 1) || (kbits == 7 && vbits == 4);
    if (qjl == 0)
        return (kbits == vbits && kbits >= 2 && kbits <= 4) || (kbits == 3 && vbits == 4);
    return false;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

uint16_t half_bits(float v) { return __half_as_ushort(__float2half_rn(v)); }

uint32_t half2_bits(float lo, float hi)
{
    return uint32_t(half_bits(lo)) | (uint32_t(half_bits(hi)) << 16);
}

int check_device(const tq_ctx* ctx)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return TQ_ERR_CUDA;
    return dev == ctx->device ? TQ_OK : TQ_ERR_DEVICE;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

tq_layout make_layout(int d, int kbits, int vbits, int qjl)
{
    tq_layout L{};
    const int w = kbits + qjl + vbits;   // bits per coordinate pair-slot of a lane string
    L.d = d;
    L.bits = vbits;
    L.m = d;
    L.kbits = kbits;
    L.vbits = vbits;
    L.tile = TQ_TILE;
    L.k_bytes_per_token = (int64_t)(kbits + qjl) * d / 8 + 2 + 2 * qjl;
    L.v_bytes_per_token = (int64_t)vbits * d / 8 + 2;
    L.tile_bytes = TQ_TILE * (L.k_bytes_per_token + L.v_bytes_per_token);
    L.code_bytes = 2LL * w * d;
    const int sb = w * d / 16;
    L.chunk_bytes = (sb % 16 == 0) ? 16 : (sb % 8 == 0) ? 8 : 4;
    L.qjl = qjl;
    return L;
}

tq_layout ctx_layout(const tq_ctx* ctx) { return make_layout(ctx->d, ctx->kbits, ctx->vbits, ctx->qjl); }

tq::Format ctx_format(const tq_ctx* ctx) { return tq::Format{ctx->d, ctx->kbits, ctx->vbits, ctx->qjl}; }

int check_cache(const tq_ctx* ctx, const tq_cache* c, int B, int Hkv)
{
    if (!c || !c->data) return TQ_ERR_INVALID_ARG;
    if (c->B != B || c->Hkv != Hkv) return TQ_ERR_INVALID_ARG;
    if (c->capacity <= 0 || c->capacity % TQ_TILE != 0) return TQ_ERR_INVALID_ARG;
    if (!aligned(c->data, 16)) return TQ_ERR_INVALID_ARG;
    (void)ctx;
    return TQ_OK;
}

// Build the device image of the tables: see tq::DevTables for the layout.
int upload_tables(tq_ctx* ctx)
{
    const auto& h = ctx->host;
    const int d = h.d, m = h.m, nk = 1 << h.kbits, nv = 1 << h.vbits;
    const float sd = std::sqrt(float(d));

    std::vector<double> bounds_k(std::max(nk, 16), 0.0), centroids_kd(std::max(nk, 16), 0.0),
        bounds_v(16, 0.0);
    for (int j = 0; j < nk; ++j) centroids_kd[j] = double(h.centroids_k[j]);
    for (int j = 0; j + 1 < nk; ++j) bounds_k[j] = double(h.bounds_k[j]);
    for (int j = 0; j + 1 < nv; ++j) bounds_v[j] = double(h.bounds_v[j]);
    std::vector<float> signs(d);
    for (int i = 0; i < d; ++i) signs[i] = float(h.signs[i]);
    // S^T as m16n8k16 B fragments: lane 4g+t of (kk, nt) holds
    // b0 = (S[8nt+g][16kk+2t], S[8nt+g][16kk+2t+1]), b1 = the same columns + 8.
    std::vector<uint2> sfrag(size_t(d / 16) * (m / 8) * 32);
    for (int kk = 0; kk < d / 16; ++kk)
        for (int nt = 0; nt < m / 8; ++nt)
            for (int lane = 0; lane < 32; ++lane) {
                const int g = lane >> 2, t = lane & 3;
                const float* row = &h.S[size_t(8 * nt + g) * d];
                const int c = 16 * kk + 2 * t;
                uint2 v;
                v.x = half2_bits(row[c], row[c + 1]);
                v.y = half2_bits(row[c + 8], row[c + 9]);
                sfrag[(size_t(kk) * (m / 8) + nt) * 32 + lane] = v;
            }
    std::vector<float> st(size_t(d) * m);
    for (int j = 0; j < m; ++j)
        for (int i = 0; i < d; ++i) st[size_t(i) * m + j] = h.S[size_t(j) * d + i];
    // Key decode table: per pair of cells, fp16x2 of both levels; for cells of
    // more than 4 bits, per cell, the level split as fp16 {hi, lo = rest}
    // (128 levels cannot all be fp16-exact under one scale).
    const bool per_code = h.kbits > 4;
    std::vector<uint32_t> lutk(per_code ? size_t(nk) : size_t(nk) * nk), lutv(size_t(nv) * nv);
    const double sdk = std::sqrt(double(d)) * double(h.alpha_k);
    if (per_code) {
        for (int f = 0; f < nk; ++f) {
            const float x = float(double(h.centroids_k[f]) * sdk);
            const float hi = __half2float(__float2half_rn(x));
            lutk[f] = half2_bits(hi, x - hi);
        }
    } else {
        for (int f = 0; f < nk * nk; ++f)
            lutk[f] = half2_bits(float(double(h.centroids_k[f & (nk - 1)]) * sdk),
                                 float(double(h.centroids_k[f >> h.kbits]) * sdk));
    }
    for (int f = 0; f < nv * nv; ++f)
        lutv[f] = half2_bits(h.centroids_v[f & (nv - 1)] * sd, h.centroids_v[f >> h.vbits] * sd);

    struct Part {
        const void* src;
        size_t bytes, off;
    };
    std::vector<Part> parts = {
        {h.centroids_k.data(), h.centroids_k.size() * 4, 0},
        {bounds_k.data(), bounds_k.size() * 8, 0},
        {centroids_kd.data(), centroids_kd.size() * 8, 0},
        {bounds_v.data(), bounds_v.size() * 8, 0},
        {signs.data(), signs.size() * 4, 0},
        {sfrag.data(), sfrag.size() * sizeof(uint2), 0},
        {st.data(), st.size() * 4, 0},
        {lutk.data(), lutk.size() * 4, 0},
        {lutv.data(), lutv.size() * 4, 0},
        {nullptr, 4, 0},  // status word
    };
    size_t total = 0;
    for (auto& p : parts) {
        p.off = total;
        total += align256(p.bytes);
    }
    void* block = nullptr;
    if (cudaMalloc(&block, total) != cudaSuccess) return TQ_ERR_CUDA;
    std::vector<uint8_t> image(total, 0);
    for (auto& p : parts)
        if (p.src) std::memcpy(image.data() + p.off, p.src, p.bytes);
    if (cudaMemcpy(block, image.data(), total, cudaMemcpyHostToDevice) != cudaSuccess) {
        cudaFree(block);
        return TQ_ERR_CUDA;
    }
    auto at = [&](int i) { return static_cast<uint8_t*>(block) + parts[i].off; };
    ctx->dev_block = block;
    tq::DevTables& t = ctx->tables;
    t.centroids_k = reinterpret_cast<const float*>(at(0));
    t.bounds_k = reinterpret_cast<const double*>(at(1));
    t.centroids_kd = reinterpret_cast<const double*>(at(2));
    t.bounds_v = reinterpret_cast<const double*>(at(3));
    t.signs = reinterpret_cast<const float*>(at(4));
    t.s_frag = reinterpret_cast<const uint2*>(at(5));
    t.s_t = reinterpret_cast<const float*>(at(6));
    t.lut_k = reinterpret_cast<const uint32_t*>(at(7));
    t.lut_v = reinterpret_cast<const uint32_t*>(at(8));
    t.status = reinterpret_cast<unsigned*>(at(9));
    t.alpha_k = h.alpha_k;
    return TQ_OK;
}

int quantize_common(tq_ctx* ctx, const void* k, const void* v, int B, int Hkv, int T,
                    const int32_t* start_pos, const tq_cache* cache, void* stream);

// tq_attend / tq_scores / tq_append_attend. With k != nullptr the T new tokens
// are appended first: inside the prologue launch when 1 <= T <= 16, else by
// the quantize kernel launched ahead of the attention launches.
int attend_common(tq_ctx* ctx, const void* q, int q_dtype, int B, int Hq, const tq_cache* cache,
                  const int32_t* seq_len, int max_len, float* out, void* ws, size_t ws_bytes,
                  void* stream, bool scores, const void* k = nullptr, const void* v = nullptr,
                  int T = 0, const int32_t* start_pos = nullptr, int cc_mode = 0)
{
    if (!ctx || !q || !seq_len || !out) return TQ_ERR_INVALID_ARG;
    if (q_dtype != TQ_DTYPE_F16 && q_dtype != TQ_DTYPE_BF16) return TQ_ERR_INVALID_ARG;
    if (B <= 0 || Hq <= 0 || !cache) return TQ_ERR_INVALID_ARG;
    int rc = check_cache(ctx, cache, B, cache->Hkv);
    if (rc) return rc;
    const int Hkv = cache->Hkv;
    if (Hkv <= 0 || Hq % Hkv != 0) return TQ_ERR_INVALID_ARG;
    if (max_len < 0 || max_len > cache->capacity) return TQ_ERR_INVALID_ARG;
    if (B > 65535 || (long long)Hkv * ((Hq / Hkv + 7) / 8) > 65535 || Hq > 65535)
        return TQ_ERR_INVALID_ARG;
    if ((rc = check_device(ctx))) return rc;
    const tq::AttendPlan plan = tq::plan_attend(ctx_format(ctx), B, Hq, Hkv, max_len, ctx->num_sms);
    if (!ws || !aligned(ws, 256)) return TQ_ERR_INVALID_ARG;
    if (ws_bytes < plan.total_bytes) return TQ_ERR_WORKSPACE;
    if (!aligned(q, 16) || !aligned(out, 16)) return TQ_ERR_INVALID_ARG;
    const bool append = k != nullptr;
    if (append) {
        if (!v || !start_pos || T < 0) return TQ_ERR_INVALID_ARG;
        if (!aligned(k, 16) || !aligned(v, 16)) return TQ_ERR_INVALID_ARG;
        if (T > 16 && (rc = quantize_common(ctx, k, v, B, Hkv, T, start_pos, cache, stream)))
            return rc;
    }
    if (scores && max_len == 0) return TQ_OK;
    tq::AttendArgs a{};
    if (append && T >= 1 && T <= 16) {
        a.k_new = static_cast<const __half*>(k);
        a.v_new = static_cast<const __half*>(v);
        a.start_pos = start_pos;
        a.T = T;
        a.cache_w = static_cast<uint8_t*>(cache->data);
    }
    a.q = q;
    a.q_bf16 = (q_dtype == TQ_DTYPE_BF16);
    a.seq_len = seq_len;
    a.cache = static_cast<const uint8_t*>(cache->data);
    a.B = B;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.capacity = cache->capacity;
    a.max_len = max_len;
    a.tile_bytes = ctx_layout(ctx).tile_bytes;
    a.qfrag = static_cast<uint32_t*>(ws);
    a.prefix = reinterpret_cast<long long*>(static_cast<uint8_t*>(ws) + align256(plan.qfrag_bytes));
    a.partial = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + align256(plan.qfrag_bytes) +
                                         align256(plan.prefix_bytes));
    a.out = out;
    a.plan = plan;
    a.cc_mode = cc_mode;
    const cudaError_t e = tq::launch_attend(ctx_format(ctx), ctx->tables, a, scores,
                                            static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

}  // namespace

extern "C" {

int tq_build_codebook(int B, int d, int codebook, float* centroids, float* bounds)
{
    if (B < 1 || B > tq::kMaxCellBits || d < 3 || d > 4096 || !centroids || !bounds)
        return TQ_ERR_INVALID_ARG;
    if (codebook == TQ_CODEBOOK_GAUSS)
        return tq::build_codebook(B, d, centroids, bounds) ? TQ_OK : TQ_ERR_CUDA;
    if (codebook == TQ_CODEBOOK_BETA)
        return tq::build_codebook_beta(B, d, centroids, bounds) ? TQ_OK : TQ_ERR_CUDA;
    return TQ_ERR_UNSUPPORTED;
}

int tq_build_tables(int d, int bits, uint64_t seed, float* centroids_k, float* bounds_k,
                    float* centroids_v, float* bounds_v, int8_t* signs, float* S)
{
    if (!supported(d, bits - 1, bits, 1)) return TQ_ERR_UNSUPPORTED;
    tq::HostTables t;
    if (!tq::build_host_tables(d, bits - 1, bits, 1, TQ_CODEBOOK_GAUSS, seed, t)) return TQ_ERR_CUDA;
    if (centroids_k) std::memcpy(centroids_k, t.centroids_k.data(), t.centroids_k.size() * 4);
    if (bounds_k) std::memcpy(bounds_k, t.bounds_k.data(), t.bounds_k.size() * 4);
    if (centroids_v) std::memcpy(centroids_v, t.centroids_v.data(), t.centroids_v.size() * 4);
    if (bounds_v) std::memcpy(bounds_v, t.bounds_v.data(), t.bounds_v.size() * 4);
    if (signs) std::memcpy(signs, t.signs.data(), t.signs.size());
    if (S) std::memcpy(S, t.S.data(), t.S.size() * 4);
    return TQ_OK;
}

int tq_init(int d, int bits, uint64_t seed, tq_ctx** out)
{
    return tq_init_ex(d, bits - 1, bits, 1, TQ_CODEBOOK_GAUSS, seed, out);
}

int tq_init_ex(int d, int kbits, int vbits, int qjl, int codebook, uint64_t seed, tq_ctx** out)
{
    if (!out) return TQ_ERR_INVALID_ARG;
    *out = nullptr;
    if (!supported(d, kbits, vbits, qjl)) return TQ_ERR_UNSUPPORTED;
    if (codebook != TQ_CODEBOOK_GAUSS && codebook != TQ_CODEBOOK_BETA) return TQ_ERR_UNSUPPORTED;
    tq_ctx* ctx = new (std::nothrow) tq_ctx();
    if (!ctx) return TQ_ERR_INVALID_ARG;
    ctx->d = d;
    ctx->bits = vbits;
    ctx->kbits = kbits;
    ctx->vbits = vbits;
    ctx->qjl = qjl;
    if (!tq::build_host_tables(d, kbits, vbits, qjl, codebook, seed, ctx->host)) {
        delete ctx;
        return TQ_ERR_CUDA;
    }
    if (cudaGetDevice(&ctx->device) != cudaSuccess ||
        cudaDeviceGetAttribute(&ctx->num_sms, cudaDevAttrMultiProcessorCount, ctx->device) !=
            cudaSuccess) {
        delete ctx;
        return TQ_ERR_CUDA;
    }
    const int rc = upload_tables(ctx);
    if (rc != TQ_OK) {
        delete ctx;
        return rc;
    }
    *out = ctx;
    return TQ_OK;
}

void tq_destroy(tq_ctx* ctx)
{
    if (!ctx) return;
    if (ctx->dev_block) {
        int prev = -1;
        cudaGetDevice(&prev);
        if (prev != ctx->device) cudaSetDevice(ctx->device);
        cudaDeviceSynchronize();
        cudaFree(ctx->dev_block);
        if (prev >= 0 && prev != ctx->device) cudaSetDevice(prev);
    }
    delete ctx;
}

int tq_cache_layout(const tq_ctx* ctx, tq_layout* out)
{
    if (!ctx || !out) return TQ_ERR_INVALID_ARG;
    *out = ctx_layout(ctx);
    return TQ_OK;
}

int tq_cache_bytes(const tq_ctx* ctx, int B, int Hkv, int capacity, size_t* bytes)
{
    if (!ctx || !bytes || B <= 0 || Hkv <= 0 || capacity <= 0 || capacity % TQ_TILE)
        return TQ_ERR_INVALID_ARG;
    *bytes = size_t(B) * Hkv * (capacity / TQ_TILE) * size_t(ctx_layout(ctx).tile_bytes);
    return TQ_OK;
}

int tq_get_tables(const tq_ctx* ctx, float* centroids_k, float* bounds_k, float* centroids_v,
                  float* bounds_v, int8_t* signs, float* S)
{
    if (!ctx) return TQ_ERR_INVALID_ARG;
    const auto& t = ctx->host;
    if (centroids_k) std::memcpy(centroids_k, t.centroids_k.data(), t.centroids_k.size() * 4);
    if (bounds_k) std::memcpy(bounds_k, t.bounds_k.data(), t.bounds_k.size() * 4);
    if (centroids_v) std::memcpy(centroids_v, t.centroids_v.data(), t.centroids_v.size() * 4);
    if (bounds_v) std::memcpy(bounds_v, t.bounds_v.data(), t.bounds_v.size() * 4);
    if (signs) std::memcpy(signs, t.signs.data(), t.signs.size());
    if (S) std::memcpy(S, t.S.data(), t.S.size() * 4);
    return TQ_OK;
}

int tq_quantize(tq_ctx* ctx, const void* k, const void* v, int B, int Hkv, int T,
                const int32_t* start_pos, const tq_cache* cache, void* stream)
{
    return quantize_common(ctx, k, v, B, Hkv, T, start_pos, cache, stream);
}

int tq_append_attend(tq_ctx* ctx, const void* q, int q_dtype, const void* k, const void* v, int B,
                     int Hq, int T, const int32_t* start_pos, const tq_cache* cache,
                     const int32_t* seq_len, int max_len, float* out, void* workspace,
                     size_t workspace_bytes, void* stream)
{
    if (!k) return TQ_ERR_INVALID_ARG;
    return attend_common(ctx, q, q_dtype, B, Hq, cache, seq_len, max_len, out, workspace,
                         workspace_bytes, stream, false, k, v, T, start_pos);
}

}  // extern "C"

namespace {

int quantize_common(tq_ctx* ctx, const void* k, const void* v, int B, int Hkv, int T,
                    const int32_t* start_pos, const tq_cache* cache, void* stream)
{
    if (!ctx || !k || !v || !start_pos) return TQ_ERR_INVALID_ARG;
    if (B <= 0 || Hkv <= 0 || T < 0 || B > 65535 || Hkv > 65535) return TQ_ERR_INVALID_ARG;
    int rc = check_cache(ctx, cache, B, Hkv);
    if (rc) return rc;
    if (!aligned(k, 16) || !aligned(v, 16)) return TQ_ERR_INVALID_ARG;
    if ((rc = check_device(ctx))) return rc;
    if (T == 0) return TQ_OK;
    tq::QuantizeArgs a{};
    a.k = static_cast<const __half*>(k);
    a.v = static_cast<const __half*>(v);
    a.start_pos = start_pos;
    a.cache = static_cast<uint8_t*>(cache->data);
    a.B = B;
    a.Hkv = Hkv;
    a.T = T;
    a.capacity = cache->capacity;
    a.tile_bytes = ctx_layout(ctx).tile_bytes;
    const cudaError_t e = tq::launch_quantize(ctx_format(ctx), ctx->tables, a,
                                              static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

}  // namespace

extern "C" {

int tq_attend_workspace(const tq_ctx* ctx, int B, int Hq, int Hkv, int max_len, size_t* bytes)
{
    if (!ctx || !bytes || B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || max_len < 0)
        return TQ_ERR_INVALID_ARG;
    *bytes = tq::plan_attend(ctx_format(ctx), B, Hq, Hkv, max_len, ctx->num_sms).total_bytes;
    return TQ_OK;
}

int tq_attend(tq_ctx* ctx, const void* q, int q_dtype, int B, int Hq, const tq_cache* cache,
              const int32_t* seq_len, int max_len, float* out, void* workspace,
              size_t workspace_bytes, void* stream)
{
    return attend_common(ctx, q, q_dtype, B, Hq, cache, seq_len, max_len, out, workspace,
                         workspace_bytes, stream, false);
}

int tq_attend_cudacore(tq_ctx* ctx, const void* q, int q_dtype, int B, int Hq, const tq_cache* cache,
                       const int32_t* seq_len, int max_len, float* out, void* workspace,
                       size_t workspace_bytes, int qjl_mode, void* stream)
{
    if (!ctx) return TQ_ERR_INVALID_ARG;
    if (ctx->d != 128 || ctx->kbits != 3 || ctx->vbits != 4 || ctx->qjl != 1) return TQ_ERR_UNSUPPORTED;
    if (qjl_mode != TQ_CC_QJL_NIBBLE && qjl_mode != TQ_CC_QJL_POPCOUNT) return TQ_ERR_INVALID_ARG;
    return attend_common(ctx, q, q_dtype, B, Hq, cache, seq_len, max_len, out, workspace,
                         workspace_bytes, stream, false, nullptr, nullptr, 0, nullptr, qjl_mode);
}

int tq_scores(tq_ctx* ctx, const void* q, int q_dtype, int B, int Hq, const tq_cache* cache,
              const int32_t* seq_len, int max_len, float* scores, void* workspace,
              size_t workspace_bytes, void* stream)
{
    return attend_common(ctx, q, q_dtype, B, Hq, cache, seq_len, max_len, scores, workspace,
                         workspace_bytes, stream, true);
}

int tq_status(tq_ctx* ctx, uint32_t* flags)
{
    if (!ctx || !flags) return TQ_ERR_INVALID_ARG;
    int rc = check_device(ctx);
    if (rc) return rc;
    if (cudaDeviceSynchronize() != cudaSuccess) return TQ_ERR_CUDA;
    if (cudaMemcpy(flags, ctx->tables.status, 4, cudaMemcpyDeviceToHost) != cudaSuccess)
        return TQ_ERR_CUDA;
    if (cudaMemset(ctx->tables.status, 0, 4) != cudaSuccess) return TQ_ERR_CUDA;
    return TQ_OK;
}

int tq_copy(const void* src, void* dst, size_t bytes, void* stream)
{
    if (!src || !dst || bytes % 16 || !aligned(src, 16) || !aligned(dst, 16))
        return TQ_ERR_INVALID_ARG;
    return tq::launch_copy(src, dst, bytes, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? TQ_OK
               : TQ_ERR_CUDA;
}

const char* tq_strerror(int code)
{
    switch (code) {
    case TQ_OK: return "ok";
    case TQ_ERR_INVALID_ARG: return "invalid argument";
    case TQ_ERR_UNSUPPORTED: return "unsupported head dimension or bit width";
    case TQ_ERR_CUDA: return "CUDA runtime error";
    case TQ_ERR_WORKSPACE: return "workspace too small";
    case TQ_ERR_DEVICE: return "called with a different device current than at tq_init";
    default: return "unknown error";
    }
}

}  // extern "C"
