// tq_attend / tq_scores / tq_append_attend kernels: split-K flash decoding
// straight from the packed cache (templates; instantiated per head dim in
// attend_d64.cu, attend_d128.cu and attend_d256.cu).
//
// The logit of query head h against cached token n is the QJL-corrected
// estimate ("[Benchmark] TurboQuant 實測：KV Cache 3-bit 壓縮，真的零損失？",
// ai-muninn.com, §"TurboQuant 是什麼：30 秒懶人包": the QJL step makes the
// attention score unbiased):
//   l_n = |k_n| (<q~, cK[idx_n]> + rho_n sqrt(pi/2)/m <S q~, 2 s_n - 1>) / sqrt(d),
// with q~ = Pi q; values stay in the rotated domain and are rotated back once
// per output: o = Pi^T sum_n softmax(l)_n |v_n| cV[vidx_n].
//
// Three kernels:
//  prologue  q~ = H (D o q) / sqrt(d) and p = S q~ per group of 8 query heads,
//            written as fp16 m16n8k16 B fragments (hi/lo; log2(e) and the
//            norms' scales folded in);
//  split     stream-K over the tiles of all (batch, kv head, group of 8 query
//            heads) units, one CTA per SM; each warp streams 16-token tiles
//            through a ring of whole-tile bulk copies, reads its own lane
//            string of each, decodes codes to fp16 tensor-core A fragments
//            through a lane-replicated shared-memory table (2 ALU ops + 1 LDS
//            per fp16x2) and sign pairs with 2 ALU ops, and runs
//              logits: [16 tok x d] x [d x 8 heads]  (codebook term)
//                      [16 tok x m] x [m x 8 heads]  (QJL sign term)
//              PV:     [d x 16 tok] x [16 tok x 8 heads]
//            on mma.sync with fp32 accumulation, with an online softmax per
//            head in registers; the warps of a CTA merge in shared memory;
//  reduce    merges the splits per query head and applies Pi^T (fp32 WHT).
// Operands come from registers because every A fragment is decoded on the
// fly; the contraction is skinny (N = 8 heads), so the legacy register-fed
// MMA fits better here than shared-memory/TMEM-fed tcgen05 tiles.
#pragma once
#include <cuda_runtime.h>
#include <math_constants.h>

#include <type_traits>
#include <utility>

#include "device_common.cuh"
#include "kernels.h"

namespace tq {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Programmatic dependent launch: every attention launch lets the next kernel in
// the stream start as soon as all of its own CTAs are running, and waits for
// its predecessor's completion (and memory) before touching anything that
// kernel may write. Without the launch attribute both are no-ops.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }

// Format (KB, VB, QJ): key cells of KB bits, value cells of VB bits, and the
// QJL sketch of the key residual (with rho) iff QJ = 1.
template <int D, int KB, int VB, int QJ>
struct AttTraits {
    static constexpr int BK = KB, BV = VB;
    static constexpr int W = KB + QJ + VB;                   // lane-string bits per pair slot
    static constexpr int KF = 2 * BK, VF = 2 * BV;          // field widths
    static constexpr int SBYTES = W * D / 16;                // bytes of a lane string
    static constexpr int CB = SBYTES % 16 == 0 ? 16 : SBYTES % 8 == 0 ? 8 : 4;
    static constexpr int NCH = SBYTES / CB;                  // chunks of a lane string
    static constexpr int NWORDS = SBYTES / 4;
    static constexpr int SBW = BK * D / 64;                  // first sign word (generic layout)
    static constexpr int VBIT0 = TileLayout<D, KB, VB, QJ>::VB0;   // first value bit
    // value pairs with two sign bits a byte ((2, 3, 1)): the QJL operands come from the value words
    static constexpr bool VSB = TileLayout<D, KB, VB, QJ>::VS_BYTES;
    static constexpr int KK = D / 16;                        // k-steps / coordinate blocks
    static constexpr int NLK = 1 << KF, NLV = 1 << VF;       // LUT entries
    static constexpr int CODE_BYTES = 2 * W * D;             // code region of a tile
    static constexpr int KNB = 32 + 32 * QJ;                 // K norm bytes of a tile
    static constexpr int TILE_BYTES = CODE_BYTES + KNB + 32;
    static constexpr int NTAB = (1 << KB) > 16 ? (1 << KB) : 16;   // key table slots of the append
    // Keys of more than 4 bits (7-bit cells, the 8-bit TurboQuant keys of
    // k8v4) are decoded code by code: a pair table would have 2^14 rows.
    static constexpr bool CK = KB > 4;
    // Byte fields: an 8-bit field that starts on a byte of the lane string (a
    // pair of 4-bit cells, or the 6-bit pair of 3-bit keys in the low bits of
    // a byte whose top bits hold two QJL signs) is turned into its table
    // offset, row * 256 + 4 * lane, by one byte permute. Such formats keep one
    // table of 256 rows of 256 bytes: the key entry, then the value entry.
    static constexpr bool PK = KB + QJ == 4;                 // keys: (3,4,1), (4,4,0)
    static_assert(!PK || !QJ || TileLayout<D, KB, VB, QJ>::KS_BYTES, "key bytes carry the signs");
    static constexpr bool PV = VB == 4;                      // values: (3,4,1), (4,4,0), (3,4,0)
    static constexpr bool ROWS = PV;
    static constexpr int LSH = ROWS ? 8 : 7;                 // log2 of a table entry's stride
    static constexpr int VW0 = VBIT0 / 32;                   // first value word (byte fields)
    // first lane-string word of the QJL sign operands: the key words (3-bit keys),
    // the value words ((2, 3, 1)), else the sign words
    static constexpr int QW0 = TileLayout<D, KB, VB, QJ>::KS_BYTES ? 0 : VSB ? VW0 : SBW;
    static_assert(!PK || ROWS, "byte-field keys come with byte-field values");
    static_assert(!CK || (ROWS && KB <= 7), "per-code keys use the row table (up to 128 codes)");
    static_assert(!PV || VBIT0 % 32 == 0, "byte-field values start on a word");
    static constexpr size_t LUT_BYTES = ROWS ? (size_t)256 * 256 : (size_t)(NLK + NLV) * 128;
    static constexpr size_t QF_BYTES = (size_t)KK * 32 * 32; // hi/lo B fragments per k-step
    static constexpr size_t SMEM_CAP = 227u * 1024u - 1024u;
    // One CTA of 16 warps per SM, 128 registers a thread: the kernel is
    // issue-bound, so warps to hide latency are worth more than registers; the
    // query fragments are read from shared memory. (Measured against 3 CTAs of
    // 4 warps with the fragments in registers at d <= 128, 8 warps at d = 256,
    // and 20 or 24 warps at d = 64: 16 warps was the fastest at every d.)
    // 8 warps where 16 rings of 2 tiles do not fit (k8v4 at d = 256).
    static constexpr int WARPS = LUT_BYTES + (size_t)16 * 2 * TILE_BYTES + QF_BYTES <= SMEM_CAP ? 16 : 8;
    static constexpr int NT = 32 * WARPS;
    static constexpr size_t MERGE_BYTES = (size_t)WARPS * 8 * (D + 2) * 4;
    static constexpr size_t QF_SMEM = QF_BYTES;
    // The decode tables are static shared arrays when they fit there (the
    // table loads then take their base as an immediate), else the front of
    // dynamic shared memory (4-bit keys with 4-bit values: 64 KB).
    static constexpr bool STATIC_LUT = LUT_BYTES <= 40 * 1024;
    // staging ring: per warp STAGES images of whole tiles, each brought in by
    // one bulk copy; 3 stages where they fit in shared memory, else 2
    static constexpr int STAGES =
        LUT_BYTES + (size_t)WARPS * 3 * TILE_BYTES + QF_SMEM <= SMEM_CAP ? 3 : 2;
    static constexpr int STAGE_BYTES = TILE_BYTES;
    static constexpr size_t RING_BYTES = (size_t)WARPS * STAGES * STAGE_BYTES;
    // dynamic shared memory: [K table][V table] (unless static), [ring, then the
    // merge buffer], [query fragments]; with an aligned row table (below):
    // [ring / merge buffer][query fragments] ... [row table at LUT_ADDR]
    static constexpr size_t BODY_BYTES = RING_BYTES > MERGE_BYTES ? RING_BYTES : MERGE_BYTES;
    // The 64 KB row table sits at shared address LUT_ADDR (64 KB-aligned) when
    // the ring, the merge buffer and the query fragments fit below it: the byte
    // permute of row_off (or the OR of lut_off) then yields the entry's full
    // shared address, and no lookup needs an add. (Measured: the adds were
    // about 65 of 464 instructions per tile.) The dynamic region then reaches
    // LUT_ADDR + 64 KB whatever the offset at which it starts.
    static constexpr uint32_t LUT_ADDR = 0x20000u;
    static constexpr bool ALIGNED = ROWS && !CK && WARPS == 16 && BODY_BYTES + QF_SMEM + 4096 <= LUT_ADDR;
    static constexpr size_t DYN_SMEM =
        ALIGNED ? (size_t)LUT_ADDR + 65536 : (STATIC_LUT ? 0 : LUT_BYTES) + BODY_BYTES + QF_SMEM;
    static_assert(LUT_BYTES + BODY_BYTES + QF_SMEM <= SMEM_CAP, "split CTA exceeds shared memory");
    static_assert(DYN_SMEM <= SMEM_CAP, "split CTA exceeds shared memory");
    static constexpr int CTAS_PER_SM = 1;
};

// Offset, inside a lane-replicated table of stride 2^SH bytes, of the entry
// selected by the F-bit field at bit `pos` of the lane string:
// field * 2^SH + 4 * lane, built with one funnel (or plain) shift and one LOP3
// (lane4 = 4 * lane occupies bits 2..6, the field bits SH and up). The
// table's own shared address is added by the load as an immediate, so no
// alignment of the table is assumed: shared memory does not start at address
// 0 of the window, and declared alignments above 1 KB are not honoured there.
template <int SH>
__device__ __forceinline__ uint32_t lut_off(const uint32_t* s, int pos, int F, uint32_t lane4)
{
    const int wi = pos >> 5, o = pos & 31;
    const uint32_t mask = ((1u << F) - 1u) << SH;
    uint32_t v;
    if (o + F <= 32)
        v = (o >= SH) ? (s[wi] >> (o - SH)) : (s[wi] << (SH - o));
    else
        v = __funnelshift_r(s[wi], s[wi + 1], o - SH);
    return (v & mask) | lane4;
}

// Offset of the row selected by byte r (0..3) of word w in a table of 256-byte
// rows: w.byte[r] * 256 + lane4, one byte permute: lane4 supplies bytes 0, 2
// and 3 (4 * lane, plus the table's shared address when that is a multiple of
// 64 KB, which makes the result the entry's full address).
__device__ __forceinline__ uint32_t row_off(uint32_t w, int r, uint32_t lane4)
{
    return __byte_perm(w, lane4, 0x7604u | ((uint32_t)r << 4));
}

// Two and four consecutive 32-bit entries at shared address x.
__device__ __forceinline__ uint2 lds64(uint32_t x)
{
    uint2 v;
    asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];\n" : "=r"(v.x), "=r"(v.y) : "r"(x));
    return v;
}
__device__ __forceinline__ uint4 lds128(uint32_t x)
{
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];\n" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(x));
    return v;
}

// A table entry: at `table` + x, or (ABS) at shared address x.
template <bool ABS = false>
__device__ __forceinline__ uint32_t lut_load(const uint32_t* table, uint32_t x)
{
    if constexpr (ABS) {
        uint32_t v;
        asm volatile("ld.shared.b32 %0, [%1];\n" : "=r"(v) : "r"(x));
        return v;
    } else {
        return *reinterpret_cast<const uint32_t*>(reinterpret_cast<const char*>(table) + x);
    }
}

// ---------------------------------------------------------------- QJL term, int8 path
// The QJL product sum_i (2 s_i - 1) x_i of a key's sign bits s_i with the
// head's projected query x = S q~ (scaled as the logits need) runs as an
// integer MMA (m16n8k32, twice the k of an fp16 MMA at the same issue cost):
// x is held as 16-bit fixed point n_i = rint(x_i / u), u = max_i |x_i| / 32767
// per head, split into a signed high byte and an unsigned low byte
// (n = 256 hi + lo); the A operand carries the signs as bytes 0 / sigma. With
// acc = sum_i sigma s_i n_i (exact in int32) and T = sum_i n_i,
//     sum_i (2 s_i - 1) x_i = u (2 acc / sigma - T) + (rounding of x, <= u/2 a term).
// Sign layouts (SL): 0 none (no QJL), 1 sign words (two bits a key pair at bits
// q and q + 16 of the pair's sign word), 2 byte fields (the two top bits of each
// key byte, or of each value byte for (2, 3, 1): token g at bit 6, token g + 8
// at bit 7).
template <int KB, int VB, int QJ>
struct SignLayout {
    static constexpr int SL =
        QJ == 0 ? 0 : (TileLayout<64, KB, VB, QJ>::KS_BYTES || TileLayout<64, KB, VB, QJ>::VS_BYTES ? 2 : 1);
};

// The coordinate held by byte i (0..3) of the B register `half` (0: b0, 1: b1)
// of lane group t in int8 k-step J: the k-positions of an A register of byte-
// field signs are the coordinates of its key word; those of sign word m are
// read with the shifts 4h + {0, 1, 2, 3} (h = J & 1), each picking one bit of
// every byte.
template <int SL>
__host__ __device__ __forceinline__ int qjl_dim(int J, int t, int half, int i)
{
    if constexpr (SL == 2)
        return 16 * (2 * J + half) + 8 * (i & 1) + 2 * t + (i >> 1);
    else
        return 16 * (4 * (J >> 1) + (J & 1) + 2 * (i & 1)) + 8 * half + 2 * t + (i >> 1);
}

// sigma of the A bytes of tokens g (sg) and g + 8 (sh)
template <int SL>
struct QjlSigma {
    static constexpr float sg = SL == 2 ? 64.f : 1.f, sh = SL == 2 ? 128.f : 1.f;
};

// A registers of int8 k-step J: a0, a2 token g, a1, a3 token g + 8 (bytes 0 / sigma).
// QW0: the first lane-string word holding the signs.
template <int SL, int QW0>
__device__ __forceinline__ void qjl_a(const uint32_t* s, int J, uint32_t (&a)[4])
{
    if constexpr (SL == 2) {
        const uint32_t w0 = s[QW0 + 2 * J], w1 = s[QW0 + 2 * J + 1];
        a[0] = w0 & 0x40404040u;
        a[1] = w0 & 0x80808080u;
        a[2] = w1 & 0x40404040u;
        a[3] = w1 & 0x80808080u;
    } else {
        const uint32_t w = s[QW0 + (J >> 1)] >> (4 * (J & 1));
        a[0] = w & 0x01010101u;
        a[1] = (w >> 1) & 0x01010101u;
        a[2] = (w >> 2) & 0x01010101u;
        a[3] = (w >> 3) & 0x01010101u;
    }
}

// Fixed-point code of x with inv = 32767 / max |x| (0 when there is no scale).
__device__ __forceinline__ int qjl_fix(float x, float inv)
{
    const int n = __float2int_rn(x * inv);
    return max(-32767, min(32767, n));
}

// ---------------------------------------------------------------- prologue
// Warp 0 of CTA (0, 0) also lays the units' tiles end to end for the split
// kernel: prefix[b] = sum over sequences b' < b of ceil(seq'/16) x units per
// sequence (seq clamped to [0, min(max_len, capacity)], flagging a clamp),
// prefix[B] = the total.
__device__ __forceinline__ void tile_prefix(const DevTables& tb, const AttendArgs& a, int lane)
{
    const int lim = min(a.max_len, a.capacity);
    const long long upb = (long long)a.Hkv * a.plan.groups;
    long long run = 0;
    bool bad = false;
    for (int b0 = 0; b0 < a.B; b0 += 32) {
        const int b = b0 + lane;
        long long v = 0;
        if (b < a.B) {
            int s = a.seq_len[b];
            if (s < 0 || s > lim) {
                bad = true;
                s = min(max(s, 0), lim);
            }
            v = (long long)((s + 15) >> 4) * upb;
        }
        long long incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long y = __shfl_up_sync(kFull, incl, o);
            if (lane >= o) incl += y;
        }
        if (b < a.B) a.prefix[b] = run + incl - v;
        run += __shfl_sync(kFull, incl, 31);
    }
    if (lane == 0) a.prefix[a.B] = run;
    if (__any_sync(kFull, bad) && lane == 0) atomicOr(tb.status, TQ_STATUS_SEQ_LEN);
}

// One CTA per (batch, kv head, group of 8 query heads): q~ = H (D o q) / sqrt(d)
// and p = S q~ for the 8 heads (S is read once per CTA), written as the fp16 B
// fragments of [log2(e) 2^7 q~ / (d alpha)] and [log2(e) 2^7 kappa p / sqrt(d)],
// each as a hi part and a lo part (x - hi), so that the two tensor-core
// products carry ~22 significant bits. alpha is the scale that makes the key
// codebook almost exact in fp16 (chosen on the host).
template <int D, int SL>
__device__ __forceinline__ void prologue_body(const DevTables& tb, const AttendArgs& a)
{
    constexpr int NT = 2 * D, VPL = D / 32;
    __shared__ float qt[D][9];          // rotated queries, [coordinate][head] (padded rows)
    __shared__ float pp[1][D][8];       // p = S q~
    __shared__ float es[8];             // per-head power-of-two scale of q~ for the split
    __shared__ float qinv[8], qu[8];    // QJL fixed point: 32767 / max |x|, and u = its inverse
    __shared__ int qsum[8];             // QJL fixed point: T = sum of the codes
    const int unit = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
    const int groups = a.plan.groups, ratio = a.Hq / a.Hkv;
    const int hkv = unit / groups, grp = unit % groups;
    const size_t units = (size_t)a.Hkv * groups;
    // The S^T fragments of this warp's two n-tiles (w, w + NT/32), requested
    // before the rotation so that their latency overlaps it (d <= 128: at
    // d = 256 they would take 64 registers, and are loaded where they are used).
    constexpr int NTW = (D / 8) / (NT / 32);   // n-tiles per warp: 2
    static_assert(NTW * (NT / 32) == D / 8, "every warp takes the same number of n-tiles");
    constexpr bool PRE = SL != 0 && D <= 128;
    uint2 bfs[PRE ? NTW : 1][D / 16];
    if constexpr (PRE) {
        const int w = tid >> 5, lane = tid & 31;
#pragma unroll
        for (int q = 0; q < NTW; ++q)
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
                bfs[q][kk] = __ldg(tb.s_frag + ((size_t)kk * (D / 8) + w + q * (NT / 32)) * 32 + lane);
    }
    if (unit == 0 && b == 0 && tid < 32) tile_prefix(tb, a, tid);

    // One warp per head: lane l holds coordinates i = 32k + l (k < D/32), so the
    // loads of q are coalesced and the transposed stores to qt hit distinct
    // banks. Walsh-Hadamard butterflies over the low five index bits run on
    // shuffles, over the high bits in-lane; then the scale 1/sqrt(d) and the
    // head's power-of-two split scale es (max |q~| es in [64, 128): the hi and
    // lo fp16 parts of q~ es below then stay clear of overflow and subnormals).
    {
        const int w = tid >> 5, lane = tid & 31;
        const float rs = rsqrtf((float)D);
        for (int h = w; h < 8; h += NT / 32) {
            const int j = grp * 8 + h;
            float x[VPL];
#pragma unroll
            for (int k = 0; k < VPL; ++k) {
                const int i = 32 * k + lane;
                x[k] = 0.f;
                if (j < ratio) {
                    const size_t off = ((size_t)b * a.Hq + hkv * ratio + j) * D + i;
                    x[k] = (a.q_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(a.q)[off])
                                     : __half2float(reinterpret_cast<const __half*>(a.q)[off])) *
                           tb.signs[i];
                }
            }
#pragma unroll
            for (int st = 1; st < 32; st <<= 1) {
#pragma unroll
                for (int k = 0; k < VPL; ++k) {
                    const float o = __shfl_xor_sync(kFull, x[k], st);
                    x[k] = (lane & st) ? (o - x[k]) : (x[k] + o);
                }
            }
#pragma unroll
            for (int st = 1; st < VPL; st <<= 1) {
#pragma unroll
                for (int k = 0; k < VPL; ++k) {
                    if (!(k & st)) {
                        const float x0 = x[k], x1 = x[k + st];
                        x[k] = x0 + x1;
                        x[k + st] = x0 - x1;
                    }
                }
            }
            float mx = 0.f;
#pragma unroll
            for (int k = 0; k < VPL; ++k) {
                x[k] *= rs;
                mx = fmaxf(mx, fabsf(x[k]));
                qt[32 * k + lane][h] = x[k];
            }
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, o));
            if (lane == 0) es[h] = (mx > 0.f && mx < 3.0e38f) ? exp2f((float)(6 - ilogbf(mx))) : 1.f;
        }
    }
    __syncthreads();
    if constexpr (SL != 0) {
    // p^T = q~^T S^T on the tensor cores: A = q~ es (rows = the 8 heads, rows
    // 8..15 zero) as hi + lo fp16 parts, B = the fp16-exact S^T fragments,
    // fp32 accumulation; warp w takes n-tiles (8 rows of S each) w, w + NW, ...
    {
        const int w = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
        const float sc = es[g];
#pragma unroll
        for (int q = 0; q < NTW; ++q) {
            const int nt = w + q * (NT / 32);
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            if constexpr (!PRE) {
                // all of this n-tile's S fragments first: one L2 round trip, not D/16
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    bfs[0][kk] = __ldg(tb.s_frag + ((size_t)kk * (D / 8) + nt) * 32 + lane);
            }
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const int c0 = 16 * kk + 2 * t;
                const float x0 = qt[c0][g] * sc, x1 = qt[c0 + 1][g] * sc;
                const float x2 = qt[c0 + 8][g] * sc, x3 = qt[c0 + 9][g] * sc;
                const float h0 = __half2float(__float2half_rn(x0)), h1 = __half2float(__float2half_rn(x1));
                const float h2 = __half2float(__float2half_rn(x2)), h3 = __half2float(__float2half_rn(x3));
                const uint2 bf = bfs[PRE ? q : 0][kk];
                mma_16816(acc, pack_half2(h0, h1), 0u, pack_half2(h2, h3), 0u, bf.x, bf.y);
                mma_16816(acc, pack_half2(x0 - h0, x1 - h1), 0u, pack_half2(x2 - h2, x3 - h3), 0u,
                          bf.x, bf.y);
            }
            // acc[0], acc[1]: head g, rows 8 nt + 2t and + 1 of S
            pp[0][8 * nt + 2 * t][g] = acc[0] / sc;
            pp[0][8 * nt + 2 * t + 1][g] = acc[1] / sc;
        }
    }
    }
    __syncthreads();
    const float scale_s = kLog2e * 128.0f * 1.2533141373155003f / ((float)D * sqrtf((float)D));
    if constexpr (SL != 0) {
        // the QJL fixed point of each head: x = p scale_s, max |x|, T = sum of the codes
        const int w = tid >> 5, lane = tid & 31;
        for (int h = w; h < 8; h += NT / 32) {
            float mx = 0.f;
            for (int i = lane; i < D; i += 32) mx = fmaxf(mx, fabsf(pp[0][i][h] * scale_s));
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, o));
            const bool ok = mx > 0.f && mx < 3.0e38f;
            const float inv = ok ? 32767.0f / mx : 0.f;
            int T = 0;
            for (int i = lane; i < D; i += 32) T += qjl_fix(pp[0][i][h] * scale_s, inv);
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) T += __shfl_xor_sync(kFull, T, o);
            if (lane == 0) {
                qinv[h] = inv;
                qu[h] = ok ? mx / 32767.0f : 0.f;
                qsum[h] = T;
            }
        }
        __syncthreads();
    }
    {
        // one codebook fragment entry (k-step, thread-in-group, head column) per thread
        const int e = tid, col = e & 7, t = (e >> 3) & 3, kk = e >> 5;
        const int c0 = 16 * kk + 2 * t;
        const int idx[4] = {c0, c0 + 1, c0 + 8, c0 + 9};
        const float scale_c = kLog2e * 128.0f / ((float)D * tb.alpha_k);
        float hv[4], lv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const float x = qt[idx[u]][col] * scale_c;
            hv[u] = __half2float(__float2half_rn(x));
            lv[u] = x - hv[u];
        }
        uint4* frag = reinterpret_cast<uint4*>(a.qfrag) + ((size_t)b * units + unit) * (D / 16) * 64;
        // codebook term: b0, b1 hi; b0, b1 lo
        frag[kk * 64 + col * 4 + t] =
            make_uint4(pack_half2(hv[0], hv[1]), pack_half2(hv[2], hv[3]), pack_half2(lv[0], lv[1]),
                       pack_half2(lv[2], lv[3]));
        if constexpr (SL != 0) {
            if (e < D) {
                // int8 k-step J, lane (col, t): b0, b1 high bytes; b0, b1 low bytes
                const int J = e >> 5, ln = e & 31, hc = ln >> 2, tt = ln & 3;
                const float inv = qinv[hc];
                uint32_t bh[2] = {0u, 0u}, bl[2] = {0u, 0u};
#pragma unroll
                for (int half = 0; half < 2; ++half) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int n = qjl_fix(pp[0][qjl_dim<SL>(J, tt, half, i)][hc] * scale_s, inv);
                        bh[half] |= ((uint32_t)(n >> 8) & 0xFFu) << (8 * i);
                        bl[half] |= ((uint32_t)n & 0xFFu) << (8 * i);
                    }
                }
                frag[J * 64 + 32 + ln] = make_uint4(bh[0], bh[1], bl[0], bl[1]);
            } else if (e < D + 32) {
                // lane ln's constants: {2u/sigma} of (g, 2t), (g, 2t+1), (g+8, 2t),
                // (g+8, 2t+1), then {-u T} of heads 2t, 2t+1
                const int ln = e - D, tt = ln & 3, h0 = 2 * tt, h1 = 2 * tt + 1;
                const float u0 = qu[h0], u1 = qu[h1];
                frag[(D / 32) * 64 + 32 + ln] =
                    make_uint4(__float_as_uint(2.f * u0 / QjlSigma<SL>::sg), __float_as_uint(2.f * u1 / QjlSigma<SL>::sg),
                               __float_as_uint(2.f * u0 / QjlSigma<SL>::sh), __float_as_uint(2.f * u1 / QjlSigma<SL>::sh));
                frag[(D / 32 + 1) * 64 + 32 + ln] =
                    make_uint4(__float_as_uint(-u0 * (float)qsum[h0]), __float_as_uint(-u1 * (float)qsum[h1]), 0u, 0u);
            }
        }
    }
}

template <int D, int SL>
__global__ void __launch_bounds__(2 * D) attend_prologue(DevTables tb, AttendArgs a)
{
    pdl_trigger();
    pdl_wait();
    prologue_body<D, SL>(tb, a);
}

// ---------------------------------------------------------------- fused append
// Bit position helpers for one token's codes inside a tile image (the tile
// layout of tq.h): a lane string is cut into chunks of CB bytes stored
// chunk-major, so string word sw of lane L sits at tile word
// ((4 sw / CB) * 32 + L) * CB/4 + (4 sw % CB) / 4.
template <int CB>
__device__ __forceinline__ int tile_word(int L, int sw)
{
    return (((4 * sw) / CB) * 32 + L) * (CB / 4) + ((4 * sw) % CB) / 4;
}

// Replace the nb-bit field at string bit `sbit` of lane L's string (a field may
// straddle two string words). Other tokens' bits in the same words may be
// written by other warps at the same time, hence the shared-memory atomics.
template <int CB>
__device__ __forceinline__ void put_field(uint32_t* img, int L, int sbit, uint32_t val, int nb)
{
    const int sw = sbit >> 5, off = sbit & 31;
    const uint32_t m = (1u << nb) - 1u;
    uint32_t* w0 = img + tile_word<CB>(L, sw);
    atomicAnd(w0, ~(m << off));
    atomicOr(w0, (val & m) << off);
    if (off + nb > 32) {
        uint32_t* w1 = img + tile_word<CB>(L, sw + 1);
        atomicAnd(w1, ~(m >> (32 - off)));
        atomicOr(w1, (val & m) >> (32 - off));
    }
}

// Quantize the T <= 16 new tokens of (sequence b, kv head hkv) exactly as
// tq_quantize does and write them into the cache: the (at most two) tiles they
// touch are copied into shared memory; each warp takes one K or V vector at a
// time (fp64 norm, sign flip, Walsh–Hadamard, cells; for keys the residual and
// its norm) and sets its bits in the tile images; then thread j computes row j
// of z = S r for every new key as an fp64 dot product (each S entry is loaded
// once for all keys) and sets the QJL sign bits s = [z >= 0]; the tiles are
// written back.
template <int D, int KB, int VB, int QJ>
__device__ __forceinline__ void append_tokens(const DevTables& tb, const AttendArgs& a, int b, int hkv,
                                              uint8_t* smem)
{
    constexpr int NT = 2 * D, NW = NT / 32, VPL = D / 32, M = D;
    using Tr = AttTraits<D, KB, VB, QJ>;
    constexpr int BK = KB, BV = VB;
    constexpr int TB = Tr::TILE_BYTES;
    constexpr int CB = Tr::CB;
    using Lay = TileLayout<D, KB, VB, QJ>;                     // field bits of a lane string
    constexpr int NB = Tr::CODE_BYTES;                        // first norm byte of a tile
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int T = a.T, start = a.start_pos[b];
    if (T <= 0) return;
    if (start < 0 || (long long)start + T > (long long)a.capacity) {
        if (tid == 0 && hkv == 0) atomicOr(tb.status, TQ_STATUS_CAPACITY);
        return;
    }
    uint32_t* img = reinterpret_cast<uint32_t*>(smem);                      // [2][TB]
    constexpr int NK = Tr::NTAB;                                              // key table slots
    double* tabs = reinterpret_cast<double*>(smem + 2 * TB);                // ck[NK] tk[NK] tv[16]
    double* rk = tabs + 2 * NK + 16;                                         // [16][D] key residuals
    double* zp = rk + 16 * D;                                                // [16][M] half-sums of z
    const int t0 = start / 16, ntile = (start + T - 1) / 16 - t0 + 1;
    uint8_t* stream = a.cache_w + ((size_t)b * a.Hkv + hkv) * (size_t)(a.capacity / 16) * TB;
    // The decode step (T = 1): this thread's first batch of S^T entries for the
    // QJL signs, requested now so that their latency overlaps the rotation.
    constexpr int SB = 32;   // S entries per batch
    constexpr bool PRE = QJ && D <= 128;   // at d = 256 the registers are short
    float sv0[PRE ? SB : 1];
    if constexpr (PRE) {
        if (T == 1) {
            const int j = tid % M, c0 = (tid / M) * (D / 2);
#pragma unroll
            for (int u = 0; u < SB; ++u) sv0[u] = __ldg(tb.s_t + (size_t)(c0 + u) * M + j);
        }
    }
    // T = 1: warp 0 quantizes the new key, warp 1 the new value; their fp16
    // coordinates are requested together with the tiles (d = 128: at d = 256
    // the registers are short)
    constexpr bool XPRE = D == 128;
    __half2 xin[XPRE ? VPL / 2 : 1];
    if (XPRE && T == 1 && w < 2) {
        const __half* src = (w == 0 ? a.k_new : a.v_new) + ((size_t)b * a.Hkv + hkv) * (size_t)D + lane * VPL;
#pragma unroll
        for (int k = 0; k < VPL; k += 2) xin[k / 2] = *reinterpret_cast<const __half2*>(src + k);
    }
    for (int e = tid; e < ntile * TB / 16; e += NT)
        reinterpret_cast<uint4*>(img)[e] = reinterpret_cast<const uint4*>(stream + (size_t)t0 * TB)[e];
    if (tid < (1 << BK)) tabs[tid] = tb.centroids_kd[tid];
    if (tid < (1 << BK) - 1) tabs[NK + tid] = tb.bounds_k[tid];
    if (tid < (1 << BV) - 1) tabs[2 * NK + tid] = tb.bounds_v[tid];
    __syncthreads();

    unsigned sat = 0u;
    const double inv_sqrt_d = 1.0 / sqrt((double)D);
#pragma unroll 1
    for (int job = w; job < 2 * T; job += NW) {
        const bool is_key = job < T;
        const int i = is_key ? job : job - T;
        const int n = start + i, tau = n & 15, g = tau & 7, half = tau >> 3;
        uint32_t* tw = img + (n / 16 - t0) * (TB / 4);
        const __half* src = (is_key ? a.k_new : a.v_new) +
                            (((size_t)b * a.Hkv + hkv) * (size_t)T + i) * D + lane * VPL;
        double x[VPL];
#pragma unroll
        for (int k = 0; k < VPL; k += 2) {
            const __half2 p = (XPRE && T == 1) ? xin[XPRE ? k / 2 : 0] : *reinterpret_cast<const __half2*>(src + k);
            x[k] = (double)__low2float(p);
            x[k + 1] = (double)__high2float(p);
        }
        double ss = 0.0;
#pragma unroll
        for (int k = 0; k < VPL; ++k) {
            ss += x[k] * x[k];
            x[k] *= (double)tb.signs[lane * VPL + k];
        }
        ss = warp_sum(ss);
        wht_warp<VPL>(x, lane);
        const double nrm = sqrt(ss);
        const double scale = nrm > 0.0 ? inv_sqrt_d / nrm : 0.0;
        if (is_key) {
            double rr = 0.0;
#pragma unroll
            for (int k = 0; k < VPL; ++k) {
                const int c = lane * VPL + k;
                const double y = x[k] * scale;
                const int idx = encode_cell<BK>(y, tabs + NK);
                if constexpr (QJ) {
                    const double r = y - tabs[idx];
                    rk[i * D + c] = r;
                    rr += r * r;
                }
                // K field: token g + 8 (r & 1), coordinate 16 kk + 8 (r >> 1) + 2 t + e
                const int kk = c >> 4, t = (c & 7) >> 1, e = c & 1;
                const int p = 4 * kk + 2 * ((c & 15) >> 3) + half;
                put_field<CB>(tw, 4 * g + t, Lay::kbit(p, e), (uint32_t)idx, BK);
            }
            if constexpr (QJ) {
                rr = warp_sum(rr);
                if (lane == 0) {
                    uint16_t* nk = reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(tw) + NB + 8 * g + 4 * half);
                    nk[0] = norm_to_half_bits(nrm, sat);
                    nk[1] = norm_to_half_bits(sqrt(rr), sat);
                }
            } else if (lane == 0) {
                *reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(tw) + NB + 4 * g + 2 * half) =
                    norm_to_half_bits(nrm, sat);
            }
        } else {
#pragma unroll
            for (int k = 0; k < VPL; ++k) {
                const int c = lane * VPL + k;
                const int idx = encode_cell<BV>(x[k] * scale, tabs + 2 * NK);
                // V field: token 2 t + 8 (r >> 1) + e, coordinate 16 kk + g' + 8 (r & 1)
                const int kk = c >> 4, gc = c & 7, t = (tau & 7) >> 1, e = tau & 1;
                const int p = 4 * kk + 2 * half + ((c & 15) >> 3);
                put_field<CB>(tw, 4 * gc + t, Lay::vbit(p, e), (uint32_t)idx, BV);
            }
            if (lane == 0)
                *reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(tw) + NB + Tr::KNB + 4 * g + 2 * half) =
                    norm_to_half_bits(nrm, sat);
        }
    }
    __syncthreads();
    // QJL signs: threads j and M + j own row j of z = S r for all new keys, each
    // summing half of the coordinates (NT = 2M); the loads of S are independent,
    // so many are in flight at once
    if constexpr (QJ) {
        const int j = tid % M, hf = tid / M;
        double z[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) z[i] = 0.0;
        if (T == 1) {   // the decode step: one key, four independent partial sums
            // the loads of S in batches of SB, all in flight at once (the first
            // batch was requested before the rotation)
            constexpr int NB = SB;
            double z1 = 0.0, z2 = 0.0, z3 = 0.0;
#pragma unroll 1
            for (int c0 = hf * (D / 2); c0 < (hf + 1) * (D / 2); c0 += NB) {
                float sv[NB];
                if (PRE && c0 == hf * (D / 2)) {
#pragma unroll
                    for (int u = 0; u < NB; ++u) sv[u] = sv0[PRE ? u : 0];
                } else {
#pragma unroll
                    for (int u = 0; u < NB; ++u) sv[u] = __ldg(tb.s_t + (size_t)(c0 + u) * M + j);
                }
#pragma unroll
                for (int u = 0; u < NB; u += 4) {
                    z[0] = fma((double)sv[u], rk[c0 + u], z[0]);
                    z1 = fma((double)sv[u + 1], rk[c0 + u + 1], z1);
                    z2 = fma((double)sv[u + 2], rk[c0 + u + 2], z2);
                    z3 = fma((double)sv[u + 3], rk[c0 + u + 3], z3);
                }
            }
            z[0] = (z[0] + z1) + (z2 + z3);
        } else {
#pragma unroll 16
            for (int c = hf * (D / 2); c < (hf + 1) * (D / 2); ++c) {
                const double sv = (double)__ldg(tb.s_t + (size_t)c * M + j);
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    if (i < T) z[i] = fma(sv, rk[i * D + c], z[i]);
            }
        }
        if (hf == 1) {
#pragma unroll
            for (int i = 0; i < 16; ++i)
                if (i < T) zp[i * M + j] = z[i];
        }
        __syncthreads();
        if (hf == 0) {
            const int kk = j >> 4, t = (j & 7) >> 1, e = j & 1;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                if (i >= T) break;
                const int n = start + i, tau = n & 15;
                const int p = 4 * kk + 2 * ((j & 15) >> 3) + (tau >> 3);
                put_field<CB>(img + (n / 16 - t0) * (TB / 4), 4 * (tau & 7) + t, Lay::sbit(p, e),
                              z[i] + zp[i * M + j] >= 0.0 ? 1u : 0u, 1);
            }
        }
    }
    __syncthreads();
    for (int e = tid; e < ntile * TB / 16; e += NT)
        reinterpret_cast<uint4*>(stream + (size_t)t0 * TB)[e] = reinterpret_cast<const uint4*>(img)[e];
    if (sat) atomicOr(tb.status, TQ_STATUS_NORM_SAT);
}

// Prologue launch of a decode step with new tokens: CTAs (x < units, b) run
// the query prologue, CTAs (units + h, b) append the new tokens of (b, kv head
// h), side by side; the split kernel, launched after this one, reads them.
template <int D, int KB, int VB, int QJ>
__global__ void __launch_bounds__(2 * D) append_prologue(DevTables tb, AttendArgs a)
{
    extern __shared__ uint4 app_smem[];
    const int units = a.Hkv * a.plan.groups;
    pdl_trigger();
    pdl_wait();
    if ((int)blockIdx.x >= units)
        append_tokens<D, KB, VB, QJ>(tb, a, blockIdx.y, blockIdx.x - units, reinterpret_cast<uint8_t*>(app_smem));
    else
        prologue_body<D, SignLayout<KB, VB, QJ>::SL>(tb, a);
}


// ---------------------------------------------------------------- reduction
// One CTA per (query head, batch): merges the partials of the CTAs whose ranges
// cover the head's unit (the range of CTA c is [c W / G, (c+1) W / G) of the W
// tiles, so tile x lies in CTA ((x + 1) G - 1) / W; a CTA with an empty range
// wrote no partial), then applies Pi^T with an fp32 Walsh-Hadamard transform.
// The partials are taken D at a time, one per thread: each thread loads one
// partial's max and sum, the block reduces them, and every thread then adds
// the chunk's rescaled accumulators of its coordinate with independent loads
// (a unit of a short batch spans many CTAs: no load waits on another).
// WHT: thread i holds coordinate i = 32 w + lane; the butterflies over the
// lane bits run on shuffles, those over the warp bits through shared memory
// (double-buffered: one barrier per stage).
template <int D>
__global__ void __launch_bounds__(D) attend_reduce(DevTables tb, AttendArgs a)
{
    constexpr int NW = D / 32;
    __shared__ float xs[2][NW][33];
    __shared__ float fsh[D];          // the chunk's partial weights exp2(m_c - M)
    __shared__ float red[2][NW];
    pdl_trigger();
    pdl_wait();
    const int hq = blockIdx.x, b = blockIdx.y, i = threadIdx.x, w = i >> 5, lane = i & 31;
    const int ratio = a.Hq / a.Hkv, groups = a.plan.groups;
    const int hkv = hq / ratio, jh = hq % ratio, grp = jh >> 3, col = jh & 7;
    const int upb = a.Hkv * groups, ju = hkv * groups + grp;
    const size_t u = (size_t)b * upb + ju;
    constexpr int RS = D + 2;
    const long long W = a.prefix[a.B], pb = a.prefix[b];
    const long long T = (a.prefix[b + 1] - pb) / upb;
    const long long G = a.plan.ctas;
    float M = -CUDART_INF_F, L = 0.f, acc = 0.f;
    if (T > 0) {   // uniform over the block
        const long long U0 = pb + ju * T, U1 = U0 + T;
        const int cf = (int)(((U0 + 1) * G - 1) / W), cl = (int)((U1 * G - 1) / W);
        const float* base = a.partial + u * 8 * RS + col * RS;   // + c * 8 * RS: slot c + u
#pragma unroll 1
        for (int c0 = cf; c0 <= cl; c0 += D) {
            const int c = c0 + i;
            float mc = -CUDART_INF_F, lc = 0.f;
            if (c <= cl && (long long)(c + 1) * W / G > (long long)c * W / G) {
                const float* ps = base + (size_t)c * 8 * RS;
                mc = ps[0];
                lc = ps[1];
            }
            float mx = mc;
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, o));
            if (lane == 0) red[0][w] = mx;
            __syncthreads();
            float Mn = M;
#pragma unroll
            for (int k = 0; k < NW; ++k) Mn = fmaxf(Mn, red[0][k]);
            // partials with max -inf (no valid token) weigh 0; so does the
            // running state while it holds nothing
            const float fo = (M == -CUDART_INF_F) ? 0.f : exp2f(M - Mn);
            const float fc = (mc == -CUDART_INF_F) ? 0.f : exp2f(mc - Mn);
            fsh[i] = fc;
            float ls = lc * fc;
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) ls += __shfl_xor_sync(kFull, ls, o);
            if (lane == 0) red[1][w] = ls;
            __syncthreads();
            float lsum = 0.f;
#pragma unroll
            for (int k = 0; k < NW; ++k) lsum += red[1][k];
            L = L * fo + lsum;
            acc *= fo;
            M = Mn;
            const int nc = min(D, cl - c0 + 1);
            const float* pc = base + (size_t)c0 * 8 * RS + 2 + i;
#pragma unroll 8
            for (int k = 0; k < nc; ++k) {
                const float f = fsh[k];
                const float v = pc[(size_t)k * 8 * RS];   // in the buffer even where unwritten
                acc = fmaf(f != 0.f ? v : 0.f, f, acc);
            }
            __syncthreads();   // fsh and red are rewritten by the next chunk
        }
    }
    float x = (L > 0.f) ? acc / L : 0.f;
#pragma unroll
    for (int st = 1; st < 32; st <<= 1) {
        const float other = __shfl_xor_sync(kFull, x, st);
        x = (lane & st) ? (other - x) : (x + other);
    }
#pragma unroll
    for (int st = 1, buf = 0; st < NW; st <<= 1, buf ^= 1) {
        xs[buf][w][lane] = x;
        __syncthreads();
        const float other = xs[buf][w ^ st][lane];
        x = (w & st) ? (other - x) : (x + other);
    }
    // Pi^T = D H / sqrt(d), and the value table carries a factor sqrt(d)
    a.out[((size_t)b * a.Hq + hq) * D + i] = x * tb.signs[i] * (1.0f / (float)D);
}

// ---------------------------------------------------------------- split kernel
// mbarrier + bulk-copy helpers (shared addresses are 32-bit).
constexpr int kWaitLimit = 1 << 22;   // bounded waits: give up and flag TQ_STATUS_WAIT_TIMEOUT

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}
// Orders this thread's earlier generic-proxy accesses of shared memory before
// later async-proxy (bulk copy) writes to it.
__device__ __forceinline__ void fence_proxy_async()
{
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}
// One bulk copy of `bytes` (a multiple of 16, both addresses 16-byte aligned)
// from global memory into this CTA's shared memory, completing on `bar`,
// whose expected transaction count is raised by the same amount.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes)
                 : "memory");
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n"
                 ::"r"(dst), "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}
// Wait for phase `parity` of `bar` to complete; false after kWaitLimit polls.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity)
{
    for (int i = 0; i < kWaitLimit; ++i) {
        uint32_t ok;
        asm volatile(
            "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
            " selp.u32 %0, 1, 0, p;\n}\n"
            : "=r"(ok)
            : "r"(bar), "r"(parity)
            : "memory");
        if (ok) return true;
    }
    return false;
}

template <int D, int KB, int VB, int QJ>
struct TileData {
    uint32_t s[AttTraits<D, KB, VB, QJ>::NWORDS];   // this lane's string of the tile
    uint2 kn;       // QJ: fp16 {|k_g|, rho_g, |k_g+8|, rho_g+8}; else .x = fp16 {|k_g|, |k_g+8|}
    uint32_t vn;    // fp16 {|v_g|, |v_g+8|}
};

template <int D, int KB, int VB, int QJ>
__device__ __forceinline__ void load_tile(const uint8_t* tp, int lane, int g, TileData<D, KB, VB, QJ>& td)
{
    using Tr = AttTraits<D, KB, VB, QJ>;
    constexpr int CB = Tr::CB, NCH = Tr::NCH;
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
        const uint8_t* src = tp + ((size_t)c * 32 + lane) * CB;
        if constexpr (CB == 16) {
            const uint4 v = __ldcs(reinterpret_cast<const uint4*>(src));
            td.s[4 * c] = v.x; td.s[4 * c + 1] = v.y; td.s[4 * c + 2] = v.z; td.s[4 * c + 3] = v.w;
        } else if constexpr (CB == 8) {
            const uint2 v = __ldcs(reinterpret_cast<const uint2*>(src));
            td.s[2 * c] = v.x; td.s[2 * c + 1] = v.y;
        } else {
            td.s[c] = __ldcs(reinterpret_cast<const uint32_t*>(src));
        }
    }
    if constexpr (QJ)
        td.kn = __ldcs(reinterpret_cast<const uint2*>(tp + Tr::CODE_BYTES + 8 * g));
    else
        td.kn.x = __ldcs(reinterpret_cast<const uint32_t*>(tp + Tr::CODE_BYTES + 4 * g));
    td.vn = __ldcs(reinterpret_cast<const uint32_t*>(tp + Tr::CODE_BYTES + Tr::KNB + 4 * g));
}

// Read this lane's bytes of a tile image in shared memory (the image has the
// cache's own layout: chunk-major lane strings, then K norms, then V norms).
template <int D, int KB, int VB, int QJ>
__device__ __forceinline__ void read_stage(const uint8_t* slot, int lane, TileData<D, KB, VB, QJ>& td)
{
    using Tr = AttTraits<D, KB, VB, QJ>;
#pragma unroll
    for (int c = 0; c < Tr::NCH; ++c) {
        const uint8_t* src = slot + (c * 32 + lane) * Tr::CB;
        if constexpr (Tr::CB == 16) {
            const uint4 v = *reinterpret_cast<const uint4*>(src);
            td.s[4 * c] = v.x; td.s[4 * c + 1] = v.y; td.s[4 * c + 2] = v.z; td.s[4 * c + 3] = v.w;
        } else if constexpr (Tr::CB == 8) {
            const uint2 v = *reinterpret_cast<const uint2*>(src);
            td.s[2 * c] = v.x; td.s[2 * c + 1] = v.y;
        } else {
            td.s[c] = *reinterpret_cast<const uint32_t*>(src);
        }
    }
    constexpr int nb = Tr::CODE_BYTES;
    const int g = lane >> 2;
    if constexpr (QJ)
        td.kn = *reinterpret_cast<const uint2*>(slot + nb + 8 * g);
    else
        td.kn.x = *reinterpret_cast<const uint32_t*>(slot + nb + 4 * g);
    td.vn = *reinterpret_cast<const uint32_t*>(slot + nb + Tr::KNB + 4 * g);
}

// Query B fragments, copied once per unit into shared memory and read from
// there by every tile (registers go to warps instead): per fp16 k-step kk the
// codebook term's x,y = hi (b0, b1), z,w = lo; per int8 k-step J < KK/2 the QJL
// term's x,y = high bytes (b0, b1), z,w = low bytes; then the lane's QJL
// constants {2u/sigma} and {-u T} (see qjl_a).
template <int KK, int NT>
struct QueryFrags {
    const uint4* sm;
    __device__ __forceinline__ void load(const uint4* src, uint4* smem, int tid)
    {
        for (int e = tid; e < KK * 64; e += NT) smem[e] = src[e];
        sm = smem;
    }
    __device__ __forceinline__ uint4 fc(int kk, int lane) const { return sm[kk * 64 + lane]; }
    __device__ __forceinline__ uint4 fs(int J, int lane) const { return sm[J * 64 + 32 + lane]; }
    __device__ __forceinline__ float4 qa(int lane) const
    {
        const uint4 v = sm[(KK / 2) * 64 + 32 + lane];
        return make_float4(__uint_as_float(v.x), __uint_as_float(v.y), __uint_as_float(v.z), __uint_as_float(v.w));
    }
    __device__ __forceinline__ float2 qb(int lane) const
    {
        const uint4 v = sm[(KK / 2 + 1) * 64 + 32 + lane];
        return make_float2(__uint_as_float(v.x), __uint_as_float(v.y));
    }
};

// The same fragments held in registers for a whole segment (loaded from the
// workspace, where the prologue wrote them): no shared-memory reads per tile,
// for 4 (KK + KK/2 + 2) registers a thread.
template <int KK, int QJ>
struct QueryFragsReg {
    uint4 c[KK];
    uint4 s[QJ ? KK / 2 : 1];
    float4 a;
    float2 bq;
    __device__ __forceinline__ void load(const uint4* src, int lane)
    {
#pragma unroll
        for (int kk = 0; kk < KK; ++kk) c[kk] = __ldg(src + kk * 64 + lane);
        if constexpr (QJ) {
#pragma unroll
            for (int J = 0; J < KK / 2; ++J) s[J] = __ldg(src + J * 64 + 32 + lane);
            const uint4 va = __ldg(src + (KK / 2) * 64 + 32 + lane);
            const uint4 vb = __ldg(src + (KK / 2 + 1) * 64 + 32 + lane);
            a = make_float4(__uint_as_float(va.x), __uint_as_float(va.y), __uint_as_float(va.z), __uint_as_float(va.w));
            bq = make_float2(__uint_as_float(vb.x), __uint_as_float(vb.y));
        }
    }
    __device__ __forceinline__ uint4 fc(int kk, int) const { return c[kk]; }
    __device__ __forceinline__ uint4 fs(int J, int) const { return s[J]; }
    __device__ __forceinline__ float4 qa(int) const { return a; }
    __device__ __forceinline__ float2 qb(int) const { return bq; }
};

// Logits (log2 units) of tokens g, g + 8 and heads 2t, 2t + 1 from the
// codebook sums (two fp32 chains: the hi and lo parts of the B operands) and the
// QJL integer sums (high, low byte chains): L = |k| (c + rho (acc u 2/sigma - u T)).
// ca, cb: the lane's QJL constants (QueryFrags::qa, qb). With OFF, the
// logits come out offset by the softmax references of heads 2t, 2t+1:
// L - m, one rounding (nm = {-m0, -m1}).
template <int QJ, bool ONE = false, bool OFF = false>
__device__ __forceinline__ void finish_logits(const uint2 kn, const float (&ah)[4], const float (&al)[4], const int (&ih)[4],
                                              const int (&il)[4], const float4 ca, const float2 cb,
                                              float (&L)[4], float2 nm = make_float2(0.f, 0.f))
{
    if constexpr (QJ) {
        const float2 kg = __half22float2(*reinterpret_cast<const __half2*>(&kn.x));   // |k_g|, rho_g
        const float2 kh = __half22float2(*reinterpret_cast<const __half2*>(&kn.y));
        const float y0 = fmaf((float)(ih[0] * 256 + il[0]), ca.x, cb.x);
        const float y1 = fmaf((float)(ih[1] * 256 + il[1]), ca.y, cb.y);
        const float y2 = fmaf((float)(ih[2] * 256 + il[2]), ca.z, cb.x);
        const float y3 = fmaf((float)(ih[3] * 256 + il[3]), ca.w, cb.y);
        const float ng = kg.x * (1.0f / 128.0f), nh = kh.x * (1.0f / 128.0f);   // the B operands carry 2^7
        const float x0 = fmaf(kg.y, y0, ONE ? ah[0] : ah[0] + al[0]);
        const float x1 = fmaf(kg.y, y1, ONE ? ah[1] : ah[1] + al[1]);
        const float x2 = fmaf(kh.y, y2, ONE ? ah[2] : ah[2] + al[2]);
        const float x3 = fmaf(kh.y, y3, ONE ? ah[3] : ah[3] + al[3]);
        if constexpr (OFF) {
            L[0] = fmaf(ng, x0, nm.x);
            L[1] = fmaf(ng, x1, nm.y);
            L[2] = fmaf(nh, x2, nm.x);
            L[3] = fmaf(nh, x3, nm.y);
        } else {
            L[0] = ng * x0;
            L[1] = ng * x1;
            L[2] = nh * x2;
            L[3] = nh * x3;
        }
    } else {
        const float2 kk2 = __half22float2(*reinterpret_cast<const __half2*>(&kn.x));
        const float ng = kk2.x * (1.0f / 128.0f), nh = kk2.y * (1.0f / 128.0f);
        const float x0 = ONE ? ah[0] : ah[0] + al[0], x1 = ONE ? ah[1] : ah[1] + al[1];
        const float x2 = ONE ? ah[2] : ah[2] + al[2], x3 = ONE ? ah[3] : ah[3] + al[3];
        if constexpr (OFF) {
            L[0] = fmaf(ng, x0, nm.x);
            L[1] = fmaf(ng, x1, nm.y);
            L[2] = fmaf(nh, x2, nm.x);
            L[3] = fmaf(nh, x3, nm.y);
        } else {
            L[0] = ng * x0;
            L[1] = ng * x1;
            L[2] = nh * x2;
            L[3] = nh * x3;
        }
    }
}

// Lazy rescale of the online softmax. The reference m of each head (the
// exponent offset of l and acc) only has to bound every logit seen so far, so
// that each p = exp2(L - m) <= 1; it need not be the running maximum. When a
// logit exceeds it, m moves to the new maximum plus this slack (log2 units),
// which makes later moves rare: for logits of unit spread, about one warp
// iteration in 16 moves it instead of one in 3. Every merge weights a partial
// by exp2(m - M), so any such bound gives the same result up to rounding.
constexpr float kRescaleSlack = 2.0f;

template <int D>
struct SplitState {
    float m0, m1, l0, l1;
    float acc[D / 16][4];
};

// Logits of one tile (log2 units) for tokens g, g+8 and heads 2t, 2t+1.
template <int D, int KB, int VB, int QJ, typename QF>
__device__ __forceinline__ void tile_logits(const TileData<D, KB, VB, QJ>& td, const QF& qf, int lane,
                                            const uint32_t* lutk, uint32_t lane4, float (&L)[4])
{
    using Tr = AttTraits<D, KB, VB, QJ>;
    constexpr int SL = SignLayout<KB, VB, QJ>::SL;
    // codebook term: two fp32 chains, the hi and lo parts of the B operands;
    // QJL term: two int8 chains, the high and low bytes of its B operands
    float ah[4], al[4];
    int ih[4] = {0, 0, 0, 0}, il[4] = {0, 0, 0, 0};
#pragma unroll
    for (int kk = 0; kk < Tr::KK; ++kk) {
        const uint4 bc = qf.fc(kk, lane);
        uint32_t ak[4], akl[4];   // akl: lo parts of per-code key levels
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int p = 4 * kk + r;
            if constexpr (Tr::PK) {
                ak[r] = lut_load<Tr::ALIGNED>(lutk, row_off(td.s[kk], r, lane4));
            } else if constexpr (Tr::CK) {
                // one table row per code, {hi, lo} of its level: the pair's hi
                // parts form the A fragment, its lo parts a second one
                using Lay = TileLayout<D, KB, VB, QJ>;
                const uint32_t e0 = lut_load<Tr::ALIGNED>(lutk, lut_off<8>(td.s, Lay::kbit(p, 0), KB, lane4));
                const uint32_t e1 = lut_load<Tr::ALIGNED>(lutk, lut_off<8>(td.s, Lay::kbit(p, 1), KB, lane4));
                ak[r] = __byte_perm(e0, e1, 0x5410u);
                akl[r] = __byte_perm(e0, e1, 0x7632u);
            } else {
                ak[r] = lut_load<Tr::ALIGNED>(lutk, lut_off<Tr::LSH>(td.s, Tr::KF * p, Tr::KF, lane4));
            }
        }
        if (kk == 0) {
            mma_16816_first(ah, ak[0], ak[1], ak[2], ak[3], bc.x, bc.y);
            mma_16816_first(al, ak[0], ak[1], ak[2], ak[3], bc.z, bc.w);
        } else {
            mma_16816(ah, ak[0], ak[1], ak[2], ak[3], bc.x, bc.y);
            mma_16816(al, ak[0], ak[1], ak[2], ak[3], bc.z, bc.w);
        }
        if constexpr (Tr::CK) mma_16816(al, akl[0], akl[1], akl[2], akl[3], bc.x, bc.y);
        if constexpr (QJ) {
            if (kk & 1) {   // one int8 k-step (32 coordinates) every second fp16 k-step
                const int J = kk >> 1;
                const uint4 bs = qf.fs(J, lane);
                uint32_t as[4];
                qjl_a<SL, Tr::QW0>(td.s, J, as);
                imma_16832<true>(ih, as[0], as[1], as[2], as[3], bs.x, bs.y);
                imma_16832<false>(il, as[0], as[1], as[2], as[3], bs.z, bs.w);
            }
        }
    }
    float4 ca = make_float4(0.f, 0.f, 0.f, 0.f);
    float2 cb = make_float2(0.f, 0.f);
    if constexpr (QJ) {
        ca = qf.qa(lane);
        cb = qf.qb(lane);
    }
    finish_logits<QJ>(td.kn, ah, al, ih, il, ca, cb, L);
}

// Online-softmax update and P V for one tile.
template <int D, int KB, int VB, int QJ>
__device__ __forceinline__ void tile_accumulate(const TileData<D, KB, VB, QJ>& td, float (&L)[4], bool v0,
                                                bool v1, const uint32_t* lutv, uint32_t lane4,
                                                SplitState<D>& st)
{
    using Tr = AttTraits<D, KB, VB, QJ>;
    // The reference of each head only moves when some logit exceeds it (rarely,
    // after the first tiles; see kRescaleSlack): only then reduce across the 8
    // token lanes and rescale. Every p = exp2(L - m) <= 1, which also keeps
    // p*|v| in fp16 range.
    const bool above = (L[0] > st.m0) || (L[2] > st.m0) || (L[1] > st.m1) || (L[3] > st.m1);
    if (__any_sync(kFull, above)) {
        float mx0 = fmaxf(L[0], L[2]), mx1 = fmaxf(L[1], L[3]);
#pragma unroll
        for (int sh = 4; sh <= 16; sh <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, sh));
            mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, sh));
        }
        const float mn0 = fmaxf(st.m0, mx0 + kRescaleSlack), mn1 = fmaxf(st.m1, mx1 + kRescaleSlack);
        const float al0 = fast_exp2(st.m0 - mn0), al1 = fast_exp2(st.m1 - mn1);
        st.l0 *= al0;
        st.l1 *= al1;
#pragma unroll
        for (int kk = 0; kk < Tr::KK; ++kk) {
            st.acc[kk][0] *= al0;
            st.acc[kk][1] *= al1;
            st.acc[kk][2] *= al0;
            st.acc[kk][3] *= al1;
        }
        st.m0 = mn0;
        st.m1 = mn1;
    }
    const float p0 = fast_exp2(L[0] - st.m0), p1 = fast_exp2(L[1] - st.m1);
    const float p2 = fast_exp2(L[2] - st.m0), p3 = fast_exp2(L[3] - st.m1);
    st.l0 += p0 + p2;
    st.l1 += p1 + p3;
    // slots past seq_len may hold anything (even NaN norms): select, never multiply
    const float2 vnf = __half22float2(*reinterpret_cast<const __half2*>(&td.vn));
    const float vn_g = v0 ? vnf.x : 0.f;
    const float vn_h = v1 ? vnf.y : 0.f;
    const uint32_t b0 = movmatrix_trans(pack_half2(p0 * vn_g, p1 * vn_g));
    const uint32_t b1 = movmatrix_trans(pack_half2(p2 * vn_h, p3 * vn_h));
#pragma unroll
    for (int kk = 0; kk < Tr::KK; ++kk) {
        uint32_t av[4];
#pragma unroll
        for (int r = 0; r < 4; ++r)
            av[r] = Tr::PV ? lut_load<Tr::ALIGNED>(lutv, row_off(td.s[Tr::VW0 + kk], r, lane4))
                           : lut_load<Tr::ALIGNED>(lutv, lut_off<Tr::LSH>(td.s, TileLayout<D, KB, VB, QJ>::vbit(4 * kk + r, 0),
                                                                          Tr::VF, lane4));
        mma_16816(st.acc[kk], av[0], av[1], av[2], av[3], b0, b1);
    }
}

// Fill the lane-replicated decode tables of a CTA of NT threads.
template <int D, int KB, int VB, int QJ, int NT>
__device__ __forceinline__ void fill_luts(const DevTables& tb, uint32_t* lutk, uint32_t* lutv, int tid)
{
    using Tr = AttTraits<D, KB, VB, QJ>;
    if constexpr (Tr::ROWS) {
        // row x: the key entry (key pair x & (NLK - 1): byte-field keys ignore
        // the sign bits above it; per-code keys: level x as fp16 hi and lo),
        // then the value entry x; 64 words a row
        for (int e = tid; e < 256 * 64; e += NT) {
            const int x = e >> 6;
            uint32_t v;
            if ((e & 63) >= 32) v = __ldg(tb.lut_v + x);
            else if (Tr::CK) v = x < (1 << KB) ? __ldg(tb.lut_k + x) : 0u;   // level x: {hi, lo}
            else v = (Tr::PK || x < Tr::NLK) ? __ldg(tb.lut_k + (x & (Tr::NLK - 1))) : 0u;
            lutk[e] = v;
        }
    } else {
        for (int e = tid; e < Tr::NLK * 32; e += NT) lutk[e] = __ldg(tb.lut_k + (e >> 5));
        for (int e = tid; e < Tr::NLV * 32; e += NT) lutv[e] = __ldg(tb.lut_v + (e >> 5));
    }
}

// Estimated logits alone: one CTA per (batch, kv head, group of 8 query heads,
// context split), every tile up to max_len, -inf past seq_len.
template <int D, int KB, int VB, int QJ>
__global__ void __launch_bounds__(AttTraits<D, KB, VB, QJ>::NT, AttTraits<D, KB, VB, QJ>::CTAS_PER_SM)
    attend_scores(DevTables tb, AttendArgs a)
{
    using Tr = AttTraits<D, KB, VB, QJ>;
    constexpr int KK = Tr::KK, WARPS = Tr::WARPS, NT = Tr::NT;
    extern __shared__ uint4 dyn_smem[];
    uint32_t* lutk;
    uint32_t* lutv;
    uint8_t* body;
    if constexpr (Tr::STATIC_LUT) {
        // two arrays, the value table first: with one combined array ptxas
        // spends about 28 more instructions per tile on the table addresses
        __shared__ __align__(16) uint32_t s_lutv[Tr::NLV * 32];
        __shared__ __align__(16) uint32_t s_lutk[Tr::NLK * 32];
        lutk = s_lutk;
        lutv = s_lutv;
        body = reinterpret_cast<uint8_t*>(dyn_smem);
    } else if constexpr (Tr::ALIGNED) {
        // the row table at shared address LUT_ADDR, the ring and fragments below it
        const uint32_t dyn_s = (uint32_t)__cvta_generic_to_shared(dyn_smem);
        lutk = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(dyn_smem) + (Tr::LUT_ADDR - dyn_s));
        lutv = lutk + 32;
        body = reinterpret_cast<uint8_t*>(dyn_smem);
    } else {
        lutk = reinterpret_cast<uint32_t*>(dyn_smem);
        lutv = lutk + (Tr::ROWS ? 32 : Tr::NLK * 32);
        body = reinterpret_cast<uint8_t*>(dyn_smem) + Tr::LUT_BYTES;
    }

    const int split = blockIdx.x, unit = blockIdx.y, b = blockIdx.z;
    const int groups = a.plan.groups;
    const int hkv = unit / groups, grp = unit % groups;
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const size_t units = (size_t)a.Hkv * groups;

    fill_luts<D, KB, VB, QJ, NT>(tb, lutk, lutv, tid);
    pdl_trigger();
    pdl_wait();
    QueryFrags<KK, NT> qf;
    qf.load(reinterpret_cast<const uint4*>(a.qfrag) + ((size_t)b * units + unit) * KK * 64,
            reinterpret_cast<uint4*>(body + Tr::BODY_BYTES), tid);
    const int seq = min(max(a.seq_len[b], 0), min(a.max_len, a.capacity));
    __syncthreads();

    const int t_begin = split * a.plan.tps;
    const int t_end = min(t_begin + a.plan.tps, a.plan.tiles);
    const uint8_t* sbase = a.cache + ((size_t)b * a.Hkv + hkv) * (size_t)(a.capacity >> 4) *
                                         (size_t)a.tile_bytes;
    // table offsets of this lane (full shared addresses with an aligned table)
    const uint32_t lane4 = (Tr::ALIGNED ? Tr::LUT_ADDR : 0u) + 4u * lane;
    const int ratio = a.Hq / a.Hkv;
    const int j0 = grp * 8 + 2 * t;
    TileData<D, KB, VB, QJ> td;
#pragma unroll 1
    for (int tl = t_begin + w; tl < t_end; tl += WARPS) {
        const int pos0 = tl * 16 + g, pos1 = pos0 + 8;
        float L[4] = {-CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F};
        if (tl * 16 < seq) {   // warp-uniform
            load_tile<D, KB, VB, QJ>(sbase + (size_t)tl * (size_t)a.tile_bytes, lane, g, td);
            tile_logits<D, KB, VB, QJ>(td, qf, lane, lutk, lane4, L);
            if (pos0 >= seq) L[0] = L[1] = -CUDART_INF_F;
            if (pos1 >= seq) L[2] = L[3] = -CUDART_INF_F;
        }
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            if (j0 + hh >= ratio) continue;
            float* row = a.out + ((size_t)b * a.Hq + hkv * ratio + j0 + hh) * a.max_len;
            if (pos0 < a.max_len) row[pos0] = L[hh] * kLn2;
            if (pos1 < a.max_len) row[pos1] = L[2 + hh] * kLn2;
        }
    }
}

// Split kernel, stream-K: the tiles of all (sequence, kv head, group of 8
// query heads) units, laid end to end (sequence b's units start at
// prefix[b]), are cut into gridDim.x equal contiguous ranges, one per CTA, so
// that one wave of CTAs does equal work whatever the lengths. A CTA walks its
// range unit by unit; for each piece (segment) its warps stream the tiles
// round-robin through per-warp rings of bulk copies, merge in shared memory and
// write one partial (m, l, acc per head) to slot CTA + unit, a slot no other
// segment uses: along the tile order both the CTA index and the unit index
// are non-decreasing and every new segment raises at least one of them.
template <int D, int KB, int VB, int QJ>
__global__ void __launch_bounds__(AttTraits<D, KB, VB, QJ>::NT, AttTraits<D, KB, VB, QJ>::CTAS_PER_SM)
    attend_split(DevTables tb, AttendArgs a)
{
    using Tr = AttTraits<D, KB, VB, QJ>;
    constexpr int KK = Tr::KK, WARPS = Tr::WARPS, NT = Tr::NT, S = Tr::STAGES;
    constexpr int RS = D + 2;
    __shared__ __align__(8) uint64_t bars[WARPS * S];   // one mbarrier per ring slot
    extern __shared__ uint4 dyn_smem[];
    // Lane-replicated decode tables: entry f of lane l at byte f*128 + 4l, so
    // the 32 lanes of a warp always hit 32 different banks.
    uint32_t* lutk;
    uint32_t* lutv;
    uint8_t* body;
    if constexpr (Tr::STATIC_LUT) {
        // two arrays, the value table first: with one combined array ptxas
        // spends about 28 more instructions per tile on the table addresses
        __shared__ __align__(16) uint32_t s_lutv[Tr::NLV * 32];
        __shared__ __align__(16) uint32_t s_lutk[Tr::NLK * 32];
        lutk = s_lutk;
        lutv = s_lutv;
        body = reinterpret_cast<uint8_t*>(dyn_smem);
    } else if constexpr (Tr::ALIGNED) {
        // the row table at shared address LUT_ADDR, the ring and fragments below it
        const uint32_t dyn_s = (uint32_t)__cvta_generic_to_shared(dyn_smem);
        lutk = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(dyn_smem) + (Tr::LUT_ADDR - dyn_s));
        lutv = lutk + 32;
        body = reinterpret_cast<uint8_t*>(dyn_smem);
    } else {
        lutk = reinterpret_cast<uint32_t*>(dyn_smem);
        lutv = lutk + (Tr::ROWS ? 32 : Tr::NLK * 32);
        body = reinterpret_cast<uint8_t*>(dyn_smem) + Tr::LUT_BYTES;
    }
    float* mrg = reinterpret_cast<float*>(body);            // [WARPS][8][D+2] after a segment
    uint4* qsm = reinterpret_cast<uint4*>(body + Tr::BODY_BYTES);

    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int c = blockIdx.x;
    const long long G = gridDim.x;
    const int groups = a.plan.groups, upb = a.Hkv * groups;
    // before the wait: only the constant tables and this CTA's own barriers
    fill_luts<D, KB, VB, QJ, NT>(tb, lutk, lutv, tid);
    // table offsets of this lane (full shared addresses with an aligned table,
    // whose value entries follow the key entries of a row at + 128)
    const uint32_t lane4 = (Tr::ALIGNED ? Tr::LUT_ADDR : 0u) + 4u * lane;
    const uint32_t lane4v = lane4 + (Tr::ALIGNED ? 128u : 0u);
    uint8_t* ring = body + (size_t)w * S * Tr::STAGE_BYTES;
    const uint32_t ring_s = (uint32_t)__cvta_generic_to_shared(ring);
    const uint32_t bar_s = (uint32_t)__cvta_generic_to_shared(bars + w * S);
    if (lane == 0) {
        for (int i = 0; i < S; ++i) mbar_init(bar_s + 8 * i, 1);
        fence_mbar_init();
    }
    __syncwarp();
    pdl_trigger();
    pdl_wait();   // the prologue's prefix and query fragments are complete from here on
    const long long W = a.prefix[a.B];
    const long long x0 = (long long)c * W / G, x1 = (long long)(c + 1) * W / G;
    if (x0 >= x1) return;   // an empty range (fewer tiles than CTAs): uniform, before any barrier
    const int lim = min(a.max_len, a.capacity);
    // Bulk copies this warp has issued / waited for (warp-uniform): copy n uses
    // ring slot n % S and completes phase (n / S) & 1 of that slot's barrier.
    uint32_t issued = 0, consumed = 0;
    bool stalled = false;   // a wait ran out: no further copies, tiles skipped
    QueryFrags<KK, NT> qf;

    // Each segment re-locates its unit from x, so that only x, x1 and the
    // partial slot stay live across the tile loop.
    long long x = x0;
#pragma unroll 1
    while (x < x1) {
        // the sequence holding tile x: the largest b with prefix[b] <= x (it has tiles)
        int b = 0;
        {
            int hi = a.B - 1;
            while (b < hi) {
                const int mid = (b + hi + 1) >> 1;
                if (a.prefix[mid] <= x) b = mid; else hi = mid - 1;
            }
        }
        const long long pb = a.prefix[b];
        const long long T = (a.prefix[b + 1] - pb) / upb;   // tiles per unit of sequence b
        const int j = (int)((x - pb) / T);
        const long long U0 = pb + (long long)j * T;
        const int sb = (int)(x - U0);
        const int se = (int)min(T, x1 - U0);
        const int seq = min(max(a.seq_len[b], 0), lim);
        const int hkv = j / groups;
        const size_t u = (size_t)b * upb + j;
        qf.load(reinterpret_cast<const uint4*>(a.qfrag) + u * KK * 64, qsm, tid);
        __syncthreads();   // tables (first segment) and query fragments visible

        const uint8_t* sbase = a.cache + ((size_t)b * a.Hkv + hkv) * (size_t)(a.capacity >> 4) *
                                             (size_t)a.tile_bytes;
        SplitState<D> st;
        st.m0 = st.m1 = -CUDART_INF_F;
        st.l0 = st.l1 = 0.f;
#pragma unroll
        for (int kk = 0; kk < KK; ++kk) st.acc[kk][0] = st.acc[kk][1] = st.acc[kk][2] = st.acc[kk][3] = 0.f;

        // Bulk-copy pipeline: S - 1 tiles of this warp are in flight while one
        // is decoded. Lane 0 issues each copy into the slot the warp finished
        // reading one iteration earlier (its values are already used).
        const int my_first = sb + w;
        fence_proxy_async();
        if (!stalled && lane == 0) {
#pragma unroll
            for (int i = 0; i < S - 1; ++i) {
                const int tl = my_first + WARPS * i;
                if (tl < se) {
                    const uint32_t sl = (issued + i) % S;
                    bulk_load(ring_s + sl * Tr::STAGE_BYTES, sbase + (size_t)tl * Tr::TILE_BYTES,
                              Tr::TILE_BYTES, bar_s + 8 * sl);
                }
            }
        }
        if (!stalled) {
#pragma unroll
            for (int i = 0; i < S - 1; ++i) issued += (my_first + WARPS * i < se) ? 1u : 0u;
        }
        TileData<D, KB, VB, QJ> td;
#pragma unroll 1
        for (int tl = my_first; tl < se && !stalled; tl += WARPS) {
            const int tn = tl + WARPS * (S - 1);
            if (tn < se) {
                fence_proxy_async();
                if (lane == 0) {
                    const uint32_t sl = issued % S;
                    bulk_load(ring_s + sl * Tr::STAGE_BYTES, sbase + (size_t)tn * Tr::TILE_BYTES,
                              Tr::TILE_BYTES, bar_s + 8 * sl);
                }
                ++issued;
            }
            const uint32_t slot = consumed % S;
            if (!mbar_wait(bar_s + 8 * slot, (consumed / S) & 1u)) {
                stalled = true;
                if (lane == 0) atomicOr(tb.status, TQ_STATUS_WAIT_TIMEOUT);
                break;
            }
            ++consumed;
            read_stage<D, KB, VB, QJ>(ring + slot * Tr::STAGE_BYTES, lane, td);
            float L[4];
            tile_logits<D, KB, VB, QJ>(td, qf, lane, lutk, lane4, L);
            const bool v0 = tl * 16 + g < seq, v1 = tl * 16 + g + 8 < seq;
            if (!v0) L[0] = L[1] = -CUDART_INF_F;
            if (!v1) L[2] = L[3] = -CUDART_INF_F;
            tile_accumulate<D, KB, VB, QJ>(td, L, v0, v1, lutv, lane4v, st);
        }

        float l0 = st.l0, l1 = st.l1;
#pragma unroll
        for (int sh = 4; sh <= 16; sh <<= 1) {
            l0 += __shfl_xor_sync(kFull, l0, sh);
            l1 += __shfl_xor_sync(kFull, l1, sh);
        }
        fence_proxy_async();
        __syncthreads();   // every warp is done with the ring: reuse it for the merge
        float* mw = mrg + (size_t)w * 8 * RS;
        if (g == 0) {
            mw[(2 * t) * RS] = st.m0;
            mw[(2 * t) * RS + 1] = l0;
            mw[(2 * t + 1) * RS] = st.m1;
            mw[(2 * t + 1) * RS + 1] = l1;
        }
#pragma unroll
        for (int kk = 0; kk < KK; ++kk) {
            mw[(2 * t) * RS + 2 + 16 * kk + g] = st.acc[kk][0];
            mw[(2 * t + 1) * RS + 2 + 16 * kk + g] = st.acc[kk][1];
            mw[(2 * t) * RS + 2 + 16 * kk + g + 8] = st.acc[kk][2];
            mw[(2 * t + 1) * RS + 2 + 16 * kk + g + 8] = st.acc[kk][3];
        }
        __syncthreads();
        float* dst = a.partial + ((size_t)c + u) * 8 * RS;
        for (int e = tid; e < 8 * RS; e += NT) {
            const int head = e / RS, col = e % RS;
            float M = -CUDART_INF_F;
#pragma unroll
            for (int ww = 0; ww < WARPS; ++ww) M = fmaxf(M, mrg[(ww * 8 + head) * RS]);
            float sum = 0.f;
            if (col == 0) {
                sum = M;
            } else {
#pragma unroll
                for (int ww = 0; ww < WARPS; ++ww) {
                    const float mwv = mrg[(ww * 8 + head) * RS];
                    if (mwv != -CUDART_INF_F) sum += mrg[(ww * 8 + head) * RS + col] * exp2f(mwv - M);
                }
            }
            dst[e] = sum;
        }
        __syncthreads();   // merge buffer and query fragments free for the next segment
        x = U0 + se;       // the next unit (or the end of the range)
    }
    // after a wait ran out: wait (bounded) for this warp's copies still in flight
    while (consumed < issued) {
        if (!mbar_wait(bar_s + 8 * (consumed % S), (consumed / S) & 1u)) break;
        ++consumed;
    }
}

// ---------------------------------------------------------------- split kernel, tile pairs
// The same computation as attend_split, with each warp taking two consecutive
// tiles per iteration: the query fragments of a k-step are read from shared
// memory once for both tiles (half the shared-memory traffic they cost), the
// two tiles' decode and MMA chains interleave, and one bulk copy brings in both
// tiles. The decode tables sit in a 64 KB region at shared address LUT_ADDR =
// 64 KB, with the query fragments and the rings of the first WA warps below it
// and the other rings (and, after a segment, the merge buffer) above it; every
// table lookup address is then one byte permute or one OR.
template <int D, int KB, int VB, int QJ>
struct PairTraits {
    using Tr = AttTraits<D, KB, VB, QJ>;
    static constexpr uint32_t LUT_ADDR = 0x10000u;
    // Query fragments in registers (12 warps of up to 168 registers) or read from
    // shared memory for every pair (16 warps of 128 registers). Measured (per
    // layer, 65K context, batch 8): registers win at d = 128 for (1, 2, 1)
    // (139 against 147 us) and (2, 3, 1) (equal; the Qwen2.5-32B-shaped 128K layer
    // 55.7 against 56.8 us), lose for (3, 4, 1) (151.4 against 148.5 us at the 70B
    // shape, 107 against 101 us at d = 64): with a quarter fewer shared-memory
    // wavefronts the kernel then waits on latency with three warps a scheduler.
    static constexpr bool FREG = D == 128 && QJ == 1 && KB <= 2;
    static constexpr int WARPS = FREG ? 12 : 16, NT = 32 * WARPS;
    using QFrag = typename std::conditional<FREG, QueryFragsReg<D / 16, QJ>, QueryFrags<D / 16, NT>>::type;
    static constexpr int PSLOT = 2 * Tr::TILE_BYTES;      // one pair of tiles
    static constexpr int RPW = 2 * PSLOT;                 // ring of one warp: two pair slots
    static constexpr size_t QF = FREG ? 0 : Tr::QF_SMEM;
    static constexpr int WA_FIT = (int)((LUT_ADDR - 4096 - QF) / RPW);
    static constexpr int WA = WA_FIT > WARPS ? WARPS : WA_FIT;   // rings below the table
    static constexpr size_t MERGE = (size_t)WARPS * 8 * (D + 2) * 4;
    static constexpr size_t ABOVE = (size_t)(WARPS - WA) * RPW > MERGE ? (size_t)(WARPS - WA) * RPW : MERGE;
    static constexpr size_t DYN_SMEM = LUT_ADDR + 65536 + ABOVE;
    static constexpr bool SUPPORTED = !Tr::CK && D <= 128 && WA >= 1 && DYN_SMEM <= Tr::SMEM_CAP;
    // the value table: in the key table's rows (+ 128 bytes) for the 256-row
    // table; else its own table at LUT_ADDR + 32 KB (aligned above its size, so
    // an OR with a field offset still yields a full address)
    static constexpr uint32_t V_OFF = Tr::ROWS ? 128u : 0x8000u;
    // Wide rows for 1- and 2-bit key cells: one byte of the key words holds
    // NRK = 4 or 2 key pairs, i.e. that many consecutive A registers of a
    // k-step, so row b of a 256-row table holds all of them (entries of
    // 4 NRK bytes, replicated over 32 / NRK lanes: an LDS.64 or LDS.128 of a
    // warp is then conflict-free) in the first 128 bytes of a 256-byte row.
    // The second 128 bytes hold the value entry: the same wide entry for
    // 2-bit values (two pairs a byte), else the 32-lane entry of field b.
    // One byte permute gives a row's full shared address.
    static constexpr bool WK = !Tr::ROWS && !Tr::CK && (KB == 1 || KB == 2);
    static constexpr int NRK = KB == 1 ? 4 : 2;
    static constexpr bool WV = WK && VB == 2;
    static_assert(Tr::ROWS || ((size_t)Tr::NLK * 128 <= 0x8000 && (size_t)Tr::NLV * 128 <= 0x8000),
                  "small tables fit their 32 KB halves");
    // lane-string words holding the key operands (codes and, byte-field keys, signs) and the values
    // (2, 3, 1): the logits' QJL operands sit in the value words, so every word is
    // staged before the logits
    static constexpr int KW0 = 0, KWN = Tr::PK ? Tr::KK : Tr::VSB ? Tr::NWORDS : Tr::VW0;
    static constexpr int VW0 = Tr::VW0, VWN = Tr::NWORDS - Tr::VW0;
};

// Words [W0, W0 + NW) of this lane's string in a tile image (chunk-major, CB-byte chunks).
template <int CB, int W0, int NW, int CAP>
__device__ __forceinline__ void stage_words(const uint8_t* slot, int lane, uint32_t (&s)[CAP])
{
    constexpr int CW = CB / 4;
#pragma unroll
    for (int c = W0 / CW; c * CW < W0 + NW; ++c) {
        const uint8_t* src = slot + (c * 32 + lane) * CB;
        uint32_t v[CW];
        if constexpr (CB == 16) {
            const uint4 x = *reinterpret_cast<const uint4*>(src);
            v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
        } else if constexpr (CB == 8) {
            const uint2 x = *reinterpret_cast<const uint2*>(src);
            v[0] = x.x; v[1] = x.y;
        } else {
            v[0] = *reinterpret_cast<const uint32_t*>(src);
        }
#pragma unroll
        for (int i = 0; i < CW; ++i)
            if (c * CW + i >= W0 && c * CW + i < W0 + NW) s[c * CW + i] = v[i];
    }
}

// Logits of two tiles (log2 units) for tokens g, g+8 and heads 2t, 2t+1; the
// query fragments of each k-step serve both tiles.
template <int D, int KB, int VB, int QJ, typename QF>
__device__ __forceinline__ void pair_logits(const TileData<D, KB, VB, QJ> (&td)[2], const QF& qf, int lane,
                                            const uint32_t* lutk, uint32_t lane4, float2 nm, float (&L)[2][4])
{
    using Tr = AttTraits<D, KB, VB, QJ>;
    constexpr int SL = SignLayout<KB, VB, QJ>::SL;
    // Codebook term: the hi and lo B parts in two accumulator chains, or, for
    // byte-field keys, in one. (Measured at (3, 4, 1), d = 128: one chain alone
    // gained nothing, the lazy rescale with offset logits alone nothing, both
    // together -2.5 % per layer; at (2, 3, 1) and (1, 2, 1) one chain cost
    // 3 % and 7 %.)
    constexpr bool ONE = Tr::PK;
    float ah[2][4], al[2][4];
    int ih[2][4] = {{0, 0, 0, 0}, {0, 0, 0, 0}}, il[2][4] = {{0, 0, 0, 0}, {0, 0, 0, 0}};
#pragma unroll
    for (int kk = 0; kk < Tr::KK; ++kk) {
        const uint4 bc = qf.fc(kk, lane);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            uint32_t ak[4];
            if constexpr (PairTraits<D, KB, VB, QJ>::WK && KB == 2) {
                // key pairs 4 kk + r: bytes 2 (kk & 1) (r = 0, 1) and + 1 (r = 2, 3) of word kk / 2
                const uint2 x0 = lds64(row_off(td[u].s[kk >> 1], 2 * (kk & 1), lane4));
                const uint2 x1 = lds64(row_off(td[u].s[kk >> 1], 2 * (kk & 1) + 1, lane4));
                ak[0] = x0.x; ak[1] = x0.y; ak[2] = x1.x; ak[3] = x1.y;
            } else if constexpr (PairTraits<D, KB, VB, QJ>::WK) {
                // key pairs 4 kk .. 4 kk + 3: byte kk & 3 of word kk / 4
                const uint4 x = lds128(row_off(td[u].s[kk >> 2], kk & 3, lane4));
                ak[0] = x.x; ak[1] = x.y; ak[2] = x.z; ak[3] = x.w;
            } else {
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const int p = 4 * kk + r;
                    if constexpr (Tr::PK)
                        ak[r] = lut_load<true>(lutk, row_off(td[u].s[kk], r, lane4));
                    else
                        ak[r] = lut_load<true>(lutk, lut_off<Tr::LSH>(td[u].s, Tr::KF * p, Tr::KF, lane4));
                }
            }
            if (kk == 0) {
                mma_16816_first(ah[u], ak[0], ak[1], ak[2], ak[3], bc.x, bc.y);
                if constexpr (ONE) mma_16816(ah[u], ak[0], ak[1], ak[2], ak[3], bc.z, bc.w);
                else mma_16816_first(al[u], ak[0], ak[1], ak[2], ak[3], bc.z, bc.w);
            } else {
                mma_16816(ah[u], ak[0], ak[1], ak[2], ak[3], bc.x, bc.y);
                mma_16816(ONE ? ah[u] : al[u], ak[0], ak[1], ak[2], ak[3], bc.z, bc.w);
            }
        }
        if constexpr (QJ) {
            if (kk & 1) {   // one int8 k-step (32 coordinates) every second fp16 k-step
                const int J = kk >> 1;
                const uint4 bs = qf.fs(J, lane);
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    uint32_t as[4];
                    qjl_a<SL, Tr::QW0>(td[u].s, J, as);
                    imma_16832<true>(ih[u], as[0], as[1], as[2], as[3], bs.x, bs.y);
                    imma_16832<false>(il[u], as[0], as[1], as[2], as[3], bs.z, bs.w);
                }
            }
        }
    }
    float4 ca = make_float4(0.f, 0.f, 0.f, 0.f);
    float2 cb = make_float2(0.f, 0.f);
    if constexpr (QJ) {
        ca = qf.qa(lane);
        cb = qf.qb(lane);
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) finish_logits<QJ, ONE, true>(td[u].kn, ah[u], al[u], ih[u], il[u], ca, cb, L[u], nm);
}

// Online-softmax update and P V for two tiles (one reference check for both).
// L holds the logits already offset by the references (L - m, see
// finish_logits). The first pair of a segment sets the references from
// scratch (m = 0 until then, with l and acc empty).
template <int D, int KB, int VB, int QJ>
__device__ __forceinline__ void pair_accumulate(const TileData<D, KB, VB, QJ> (&td)[2], float (&L)[2][4],
                                                uint32_t lane4v, SplitState<D>& st, bool first)
{
    using Tr = AttTraits<D, KB, VB, QJ>;
    const bool above = (L[0][0] > 0.f) || (L[0][2] > 0.f) || (L[0][1] > 0.f) || (L[0][3] > 0.f) ||
                       (L[1][0] > 0.f) || (L[1][2] > 0.f) || (L[1][1] > 0.f) || (L[1][3] > 0.f);
    if (__any_sync(kFull, above) || first) {
        float mx0 = fmaxf(fmaxf(L[0][0], L[0][2]), fmaxf(L[1][0], L[1][2]));
        float mx1 = fmaxf(fmaxf(L[0][1], L[0][3]), fmaxf(L[1][1], L[1][3]));
#pragma unroll
        for (int sh = 4; sh <= 16; sh <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, sh));
            mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, sh));
        }
        // the references move up by d (every pair holds a valid token, so mx is finite)
        const float d0 = first ? mx0 + kRescaleSlack : fmaxf(mx0 + kRescaleSlack, 0.f);
        const float d1 = first ? mx1 + kRescaleSlack : fmaxf(mx1 + kRescaleSlack, 0.f);
        const float al0 = first ? 0.f : fast_exp2(-d0), al1 = first ? 0.f : fast_exp2(-d1);
        st.l0 *= al0;
        st.l1 *= al1;
#pragma unroll
        for (int kk = 0; kk < Tr::KK; ++kk) {
            st.acc[kk][0] *= al0;
            st.acc[kk][1] *= al1;
            st.acc[kk][2] *= al0;
            st.acc[kk][3] *= al1;
        }
        st.m0 += d0;
        st.m1 += d1;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            L[u][0] -= d0;
            L[u][2] -= d0;
            L[u][1] -= d1;
            L[u][3] -= d1;
        }
    }
    uint32_t b0[2], b1[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const float p0 = fast_exp2(L[u][0]), p1 = fast_exp2(L[u][1]);
        const float p2 = fast_exp2(L[u][2]), p3 = fast_exp2(L[u][3]);
        st.l0 += p0 + p2;
        st.l1 += p1 + p3;
        // masked tokens carry |v| = +0 (set by the caller)
        const float2 vnf = __half22float2(*reinterpret_cast<const __half2*>(&td[u].vn));
        b0[u] = movmatrix_trans(pack_half2(p0 * vnf.x, p1 * vnf.x));
        b1[u] = movmatrix_trans(pack_half2(p2 * vnf.y, p3 * vnf.y));
    }
#pragma unroll
    for (int kk = 0; kk < Tr::KK; ++kk) {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            uint32_t av[4];
            if constexpr (PairTraits<D, KB, VB, QJ>::WV) {
                // value pairs 4 kk + j: bytes 2 (kk & 1) (j = 0, 1) and + 1 of value word kk / 2
                const uint32_t w = td[u].s[Tr::VW0 + (kk >> 1)];
                const uint2 x0 = lds64(row_off(w, 2 * (kk & 1), lane4v));
                const uint2 x1 = lds64(row_off(w, 2 * (kk & 1) + 1, lane4v));
                av[0] = x0.x; av[1] = x0.y; av[2] = x1.x; av[3] = x1.y;
            } else {
                constexpr int VSH = PairTraits<D, KB, VB, QJ>::WK ? 8 : Tr::LSH;   // row stride
#pragma unroll
                for (int r = 0; r < 4; ++r)
                    av[r] = (Tr::PV || Tr::VSB)
                                ? lut_load<true>(nullptr, row_off(td[u].s[Tr::VW0 + kk], r, lane4v))
                                : lut_load<true>(nullptr, lut_off<VSH>(td[u].s, Tr::VBIT0 + Tr::VF * (4 * kk + r),
                                                                          Tr::VF, lane4v));
            }
            mma_16816(st.acc[kk], av[0], av[1], av[2], av[3], b0[u], b1[u]);
        }
    }
}

template <int D, int KB, int VB, int QJ>
__global__ void __launch_bounds__(PairTraits<D, KB, VB, QJ>::NT, 1) attend_split2(DevTables tb, AttendArgs a)
{
    using Tr = AttTraits<D, KB, VB, QJ>;
    using P2 = PairTraits<D, KB, VB, QJ>;
    constexpr int KK = Tr::KK, WARPS = P2::WARPS, NT = P2::NT, TB = Tr::TILE_BYTES, CB = Tr::CB;
    constexpr int RS = D + 2;
    __shared__ __align__(8) uint64_t bars[WARPS * 2];   // one mbarrier per pair slot
    extern __shared__ uint4 dyn_smem[];
    uint8_t* dyn = reinterpret_cast<uint8_t*>(dyn_smem);
    const uint32_t dyn_s = (uint32_t)__cvta_generic_to_shared(dyn_smem);
    uint32_t* lutk = reinterpret_cast<uint32_t*>(dyn + (P2::LUT_ADDR - dyn_s));
    uint32_t* lutv = lutk + P2::V_OFF / 4;
    uint8_t* above = dyn + (P2::LUT_ADDR + 65536 - dyn_s);
    uint4* qsm = reinterpret_cast<uint4*>(dyn);
    float* mrg = reinterpret_cast<float*>(above);         // [WARPS][8][D+2] after a segment

    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int c = blockIdx.x;
    const long long G = gridDim.x;
    const int groups = a.plan.groups, upb = a.Hkv * groups;
    if constexpr (P2::WK) {
        // 256 rows of 64 words: key entry of byte x (NRK words, 32 / NRK replicas), then the
        // value entry (2-bit values: two words, 16 replicas; else field x, 32 replicas)
        constexpr int FK = 2 * KB;
        for (int e = tid; e < 256 * 64; e += NT) {
            const int x = e >> 6, col = e & 63;
            uint32_t v;
            if (col < 32) {
                const int i = col % P2::NRK;
                v = __ldg(tb.lut_k + ((x >> (FK * i)) & ((1 << FK) - 1)));
            } else if constexpr (P2::WV) {
                v = __ldg(tb.lut_v + ((x >> (4 * (col & 1))) & 15));
            } else if constexpr (Tr::VSB) {
                v = __ldg(tb.lut_v + (x & (Tr::NLV - 1)));   // value pair in bits 0..5, signs above
            } else {
                v = x < Tr::NLV ? __ldg(tb.lut_v + x) : 0u;
            }
            lutk[e] = v;
        }
    } else {
        fill_luts<D, KB, VB, QJ, NT>(tb, lutk, lutv, tid);
    }
    // full shared addresses of this lane's table entries
    const uint32_t lane4 = P2::WK ? P2::LUT_ADDR + (uint32_t)(lane % (32 / P2::NRK)) * (4u * P2::NRK)
                                  : P2::LUT_ADDR + 4u * lane;
    const uint32_t lane4v = P2::WK ? (P2::WV ? P2::LUT_ADDR + 128u + (uint32_t)(lane & 15) * 8u
                                             : P2::LUT_ADDR + 128u + 4u * lane)
                                   : lane4 + P2::V_OFF;
    uint8_t* ring = w < P2::WA ? dyn + P2::QF + (size_t)w * P2::RPW : above + (size_t)(w - P2::WA) * P2::RPW;
    const uint32_t ring_s = (uint32_t)__cvta_generic_to_shared(ring);
    const uint32_t bar_s = (uint32_t)__cvta_generic_to_shared(bars + w * 2);
    if (lane == 0) {
        mbar_init(bar_s, 1);
        mbar_init(bar_s + 8, 1);
        fence_mbar_init();
    }
    __syncwarp();
    pdl_trigger();
    pdl_wait();   // the prologue's prefix and query fragments are complete from here on
    const long long W = a.prefix[a.B];
    const long long x0 = (long long)c * W / G, x1 = (long long)(c + 1) * W / G;
    if (x0 >= x1) return;   // an empty range (fewer tiles than CTAs): uniform, before any barrier
    const int lim = min(a.max_len, a.capacity);
    // Pair copies this warp has issued / waited for (warp-uniform): copy n uses
    // slot n % 2 and completes phase (n / 2) & 1 of that slot's barrier.
    uint32_t issued = 0, consumed = 0;
    bool stalled = false;
    typename P2::QFrag qf;

    long long x = x0;
#pragma unroll 1
    while (x < x1) {
        int b = 0;
        {
            int hi = a.B - 1;
            while (b < hi) {
                const int mid = (b + hi + 1) >> 1;
                if (a.prefix[mid] <= x) b = mid; else hi = mid - 1;
            }
        }
        const long long pb = a.prefix[b];
        const long long T = (a.prefix[b + 1] - pb) / upb;
        const int j = (int)((x - pb) / T);
        const long long U0 = pb + (long long)j * T;
        const int sb = (int)(x - U0);
        const int se = (int)min(T, x1 - U0);
        const int seq = min(max(a.seq_len[b], 0), lim);
        const int hkv = j / groups;
        const size_t u = (size_t)b * upb + j;
        const uint8_t* sbase = a.cache + ((size_t)b * a.Hkv + hkv) * (size_t)(a.capacity >> 4) *
                                             (size_t)a.tile_bytes;
        // pair p of the segment: tiles sb + 2p and sb + 2p + 1 (the last pair may hold one).
        // The warp's first pair is requested before the query fragments are read,
        // so that the two latencies overlap (the ring is apart from the fragment
        // and table regions, and the previous segment's merge ended in a barrier).
        const int ntile = se - sb, npair = (ntile + 1) >> 1;
        fence_proxy_async();
        if (!stalled && w < npair) {
            if (lane == 0) {
                const int n = min(2, ntile - 2 * w);
                const uint32_t sl = issued & 1u;
                bulk_load(ring_s + sl * P2::PSLOT, sbase + (size_t)(sb + 2 * w) * TB, (uint32_t)(n * TB),
                          bar_s + 8 * sl);
            }
            ++issued;
        }
        if constexpr (P2::FREG)
            qf.load(reinterpret_cast<const uint4*>(a.qfrag) + u * KK * 64, lane);
        else
            qf.load(reinterpret_cast<const uint4*>(a.qfrag) + u * KK * 64, qsm, tid);
        __syncthreads();   // tables (first segment) and query fragments visible

        SplitState<D> st;
        st.m0 = st.m1 = 0.f;   // set by the warp's first pair (see pair_accumulate)
        st.l0 = st.l1 = 0.f;
#pragma unroll
        for (int kk = 0; kk < KK; ++kk) st.acc[kk][0] = st.acc[kk][1] = st.acc[kk][2] = st.acc[kk][3] = 0.f;
        TileData<D, KB, VB, QJ> td[2];
#pragma unroll 1
        for (int p = w; p < npair && !stalled; p += WARPS) {
            const int pn = p + WARPS;
            if (pn < npair) {
                fence_proxy_async();
                if (lane == 0) {
                    const int n = min(2, ntile - 2 * pn);
                    const uint32_t sl = issued & 1u;
                    bulk_load(ring_s + sl * P2::PSLOT, sbase + (size_t)(sb + 2 * pn) * TB, (uint32_t)(n * TB),
                              bar_s + 8 * sl);
                }
                ++issued;
            }
            const uint32_t slot = consumed & 1u;
            if (!mbar_wait(bar_s + 8 * slot, (consumed >> 1) & 1u)) {
                stalled = true;
                if (lane == 0) atomicOr(tb.status, TQ_STATUS_WAIT_TIMEOUT);
                break;
            }
            ++consumed;
            const uint8_t* sp = ring + slot * P2::PSLOT;
            const int tl0 = sb + 2 * p;
            const bool two = 2 * p + 1 < ntile;
            // key words and norms of both tiles (a missing second tile reads stale
            // bytes of the slot: every table index stays in range and it is masked)
#pragma unroll
            for (int uu = 0; uu < 2; ++uu) {
                const uint8_t* tp = sp + uu * TB;
                stage_words<CB, P2::KW0, P2::KWN, Tr::NWORDS>(tp, lane, td[uu].s);
                if constexpr (QJ)
                    td[uu].kn = *reinterpret_cast<const uint2*>(tp + Tr::CODE_BYTES + 8 * g);
                else
                    td[uu].kn.x = *reinterpret_cast<const uint32_t*>(tp + Tr::CODE_BYTES + 4 * g);
                td[uu].vn = *reinterpret_cast<const uint32_t*>(tp + Tr::CODE_BYTES + Tr::KNB + 4 * g);
            }
            float L[2][4];
            pair_logits<D, KB, VB, QJ>(td, qf, lane, lutk, lane4, make_float2(-st.m0, -st.m1), L);
            // Tokens at or past seq_len (only in a unit's last pair, or a missing
            // second tile): logit -inf and value norm +0. Their slots may hold
            // anything, NaN norms included: select, never multiply.
            if (!(two && (tl0 + 2) * 16 <= seq)) {   // warp-uniform
#pragma unroll
                for (int uu = 0; uu < 2; ++uu) {
                    const int base = (tl0 + uu) * 16 + g;
                    const bool ok = uu == 0 || two;
                    if (!(ok && base < seq)) {
                        L[uu][0] = L[uu][1] = -CUDART_INF_F;
                        td[uu].vn &= 0xFFFF0000u;
                    }
                    if (!(ok && base + 8 < seq)) {
                        L[uu][2] = L[uu][3] = -CUDART_INF_F;
                        td[uu].vn &= 0x0000FFFFu;
                    }
                }
            }
            if constexpr (!Tr::VSB) {
#pragma unroll
                for (int uu = 0; uu < 2; ++uu)
                    stage_words<CB, P2::VW0, P2::VWN, Tr::NWORDS>(sp + uu * TB, lane, td[uu].s);
            }
            pair_accumulate<D, KB, VB, QJ>(td, L, lane4v, st, p == w);
        }

        float l0 = st.l0, l1 = st.l1;
#pragma unroll
        for (int sh = 4; sh <= 16; sh <<= 1) {
            l0 += __shfl_xor_sync(kFull, l0, sh);
            l1 += __shfl_xor_sync(kFull, l1, sh);
        }
        fence_proxy_async();
        __syncthreads();   // every warp is done with its ring: reuse the upper rings for the merge
        float* mw = mrg + (size_t)w * 8 * RS;
        if (g == 0) {
            const bool idle = w >= npair;   // no pair: no reference, the merge skips it
            mw[(2 * t) * RS] = idle ? -CUDART_INF_F : st.m0;
            mw[(2 * t) * RS + 1] = l0;
            mw[(2 * t + 1) * RS] = idle ? -CUDART_INF_F : st.m1;
            mw[(2 * t + 1) * RS + 1] = l1;
        }
#pragma unroll
        for (int kk = 0; kk < KK; ++kk) {
            mw[(2 * t) * RS + 2 + 16 * kk + g] = st.acc[kk][0];
            mw[(2 * t + 1) * RS + 2 + 16 * kk + g] = st.acc[kk][1];
            mw[(2 * t) * RS + 2 + 16 * kk + g + 8] = st.acc[kk][2];
            mw[(2 * t + 1) * RS + 2 + 16 * kk + g + 8] = st.acc[kk][3];
        }
        __syncthreads();
        float* dst = a.partial + ((size_t)c + u) * 8 * RS;
        for (int e = tid; e < 8 * RS; e += NT) {
            const int head = e / RS, col = e % RS;
            float M = -CUDART_INF_F;
#pragma unroll
            for (int ww = 0; ww < WARPS; ++ww) M = fmaxf(M, mrg[(ww * 8 + head) * RS]);
            float sum = 0.f;
            if (col == 0) {
                sum = M;
            } else {
#pragma unroll
                for (int ww = 0; ww < WARPS; ++ww) {
                    const float mwv = mrg[(ww * 8 + head) * RS];
                    if (mwv != -CUDART_INF_F) sum += mrg[(ww * 8 + head) * RS + col] * exp2f(mwv - M);
                }
            }
            dst[e] = sum;
        }
        __syncthreads();   // merge buffer and query fragments free for the next segment
        x = U0 + se;
    }
    // after a wait ran out: wait (bounded) for this warp's copies still in flight
    while (consumed < issued) {
        if (!mbar_wait(bar_s + 8 * (consumed & 1u), (consumed >> 1) & 1u)) break;
        ++consumed;
    }
}

#include "attend_cc.cuh"

// cudaFuncSetAttribute once per (kernel, device).
template <typename K>
cudaError_t allow_smem(K kernel, size_t bytes, unsigned long long& done_mask)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = 1ull << (dev & 63);
    if (__atomic_load_n(&done_mask, __ATOMIC_ACQUIRE) & bit) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess) __atomic_fetch_or(&done_mask, bit, __ATOMIC_ACQ_REL);
    return e;
}

// Launch with the programmatic-stream-serialization attribute (see pdl_wait).
template <typename... P, typename... A>
cudaError_t launch_pdl(void (*kern)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       A&&... args)
{
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
    return cudaLaunchKernelEx(&cfg, kern, std::forward<A>(args)...);
}

template <int D, int KB, int VB, int QJ>
cudaError_t launch_attend_t(const DevTables& tb, const AttendArgs& a, bool scores, cudaStream_t st)
{
    using Tr = AttTraits<D, KB, VB, QJ>;
    static unsigned long long done_scores = 0, done_attend = 0;
    if (a.tile_bytes != Tr::TILE_BYTES) return cudaErrorInvalidValue;   // the bulk copies' size
    const int units = a.Hkv * a.plan.groups;
    cudaError_t e;
    if (a.k_new != nullptr && a.T > 0) {
        static unsigned long long done_append = 0;
        constexpr int TB = Tr::TILE_BYTES;
        const size_t smem = 2 * (size_t)TB + 8 * (2 * (size_t)Tr::NTAB + 16 + (size_t)16 * D + (size_t)16 * D);
        auto kern = append_prologue<D, KB, VB, QJ>;
        if ((e = allow_smem(kern, smem, done_append)) != cudaSuccess) return e;
        e = launch_pdl(kern, dim3(units + a.Hkv, a.B), dim3(2 * D), smem, st, tb, a);
    } else {
        e = launch_pdl(attend_prologue<D, SignLayout<KB, VB, QJ>::SL>, dim3(units, a.B), dim3(2 * D), 0, st, tb, a);
    }
    if (e != cudaSuccess) return e;
    if (scores) {
        auto kern = attend_scores<D, KB, VB, QJ>;
        if ((e = allow_smem(kern, Tr::DYN_SMEM, done_scores)) != cudaSuccess) return e;
        if (a.plan.tiles > 0)
            e = launch_pdl(kern, dim3(a.plan.nsplit, units, a.B), dim3(Tr::NT), Tr::DYN_SMEM, st, tb, a);
        return e;
    }
    if (a.cc_mode != 0) {
        if constexpr (D == CcTraits::D && KB == CcTraits::KB && VB == CcTraits::VB && QJ == CcTraits::QJ) {
            static unsigned long long done_cc1 = 0, done_cc2 = 0;
            auto kern = a.cc_mode == 2 ? attend_cc<2> : attend_cc<1>;
            if ((e = allow_smem(kern, CcTraits::SMEM, a.cc_mode == 2 ? done_cc2 : done_cc1)) != cudaSuccess)
                return e;
            if (a.plan.tiles > 0 &&
                (e = launch_pdl(kern, dim3(a.plan.ctas), dim3(CcTraits::NT), CcTraits::SMEM, st, tb, a)) !=
                    cudaSuccess)
                return e;
            return launch_pdl(attend_reduce<D>, dim3(a.Hq, a.B), dim3(D), 0, st, tb, a);
        } else {
            return cudaErrorNotSupported;
        }
    }
    if constexpr (PairTraits<D, KB, VB, QJ>::SUPPORTED) {
        using P2 = PairTraits<D, KB, VB, QJ>;
        auto kern = attend_split2<D, KB, VB, QJ>;
        if ((e = allow_smem(kern, P2::DYN_SMEM, done_attend)) != cudaSuccess) return e;
        if (a.plan.tiles > 0 &&
            (e = launch_pdl(kern, dim3(a.plan.ctas), dim3(P2::NT), P2::DYN_SMEM, st, tb, a)) != cudaSuccess)
            return e;
    } else {
        auto kern = attend_split<D, KB, VB, QJ>;
        if ((e = allow_smem(kern, Tr::DYN_SMEM, done_attend)) != cudaSuccess) return e;
        if (a.plan.tiles > 0 &&
            (e = launch_pdl(kern, dim3(a.plan.ctas), dim3(Tr::NT), Tr::DYN_SMEM, st, tb, a)) != cudaSuccess)
            return e;
    }
    return launch_pdl(attend_reduce<D>, dim3(a.Hq, a.B), dim3(D), 0, st, tb, a);
}

}  // namespace
}  // namespace tq
