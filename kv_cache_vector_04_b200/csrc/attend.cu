// Host side of the attention launches: the work plan, the dispatch to the
// per-head-dim launch tables, and the streaming copy kernel that measures HBM
// bandwidth in the same process.
#include "attend_impl.cuh"

namespace tq {
namespace {

__global__ void copy_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, size_t n)
{
    size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    for (; i < n; i += stride) __stcs(dst + i, __ldcs(src + i));
}

}  // namespace

int attend_ctas_per_sm(const Format& f)
{
#define TQ_C(DD, KB, VB, QJ) \
    if (f.d == DD && f.kb == KB && f.vb == VB && f.qjl == QJ) return AttTraits<DD, KB, VB, QJ>::CTAS_PER_SM;
    TQ_FORMATS(TQ_C)
#undef TQ_C
    return 1;
}

AttendPlan plan_attend(const Format& f, int B, int Hq, int Hkv, int max_len, int num_sms)
{
    const int d = f.d;
    AttendPlan p{};
    const int ratio = Hq / Hkv;
    p.groups = (ratio + 7) / 8;
    const long long units = (long long)B * Hkv * p.groups;
    p.tiles = (max_len + 15) / 16;
    // tq_scores: one CTA per (unit, context split), about two waves
    const long long per_sm = attend_ctas_per_sm(f);
    const long long target = 2 * per_sm * num_sms;
    long long ns = (target + units - 1) / units;
    const long long max_ns = (p.tiles + 15) / 16;      // at least 16 tiles (2 per warp) per split
    if (ns > max_ns) ns = max_ns;
    if (ns < 1) ns = 1;
    p.tps = p.tiles > 0 ? (int)((p.tiles + ns - 1) / ns) : 0;
    p.nsplit = p.tps > 0 ? (p.tiles + p.tps - 1) / p.tps : 1;
    // tq_attend: stream-K, one wave of CTAs (fewer when there are under 16 tiles per CTA)
    long long ctas = per_sm * num_sms;
    const long long most = (units * p.tiles + 15) / 16;
    if (ctas > most) ctas = most;
    if (ctas < 1) ctas = 1;
    p.ctas = (int)ctas;
    p.qfrag_bytes = (size_t)units * (d / 16) * 32 * 32;
    p.prefix_bytes = (size_t)(B + 1) * sizeof(long long);
    p.partial_bytes = (size_t)(ctas + units) * 8 * (d + 2) * sizeof(float);
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    p.total_bytes = up(p.qfrag_bytes) + up(p.prefix_bytes) + up(p.partial_bytes);
    return p;
}

cudaError_t launch_attend(const Format& f, const DevTables& tb, const AttendArgs& a, bool scores,
                          cudaStream_t st)
{
    switch (f.d) {
    case 64: return launch_attend_d64(f, tb, a, scores, st);
    case 128: return launch_attend_d128(f, tb, a, scores, st);
    case 256: return launch_attend_d256(f, tb, a, scores, st);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_copy(const void* src, void* dst, size_t bytes, cudaStream_t st)
{
    const size_t n = bytes / 16;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    size_t blocks = (n + 255) / 256;
    const size_t cap = (size_t)sms * 8;
    if (blocks > cap) blocks = cap;
    if (blocks == 0) return cudaSuccess;
    copy_kernel<<<(unsigned)blocks, 256, 0, st>>>(reinterpret_cast<const uint4*>(src),
                                                  reinterpret_cast<uint4*>(dst), n);
    return cudaGetLastError();
}

}  // namespace tq
