// tq_quantize, fast path: full 16-token tiles at d <= 128 with cells of at
// most 4 bits, one warp per tile, everything in registers.
//
// The arithmetic is that of quantize_kernel (the pages' steps: rotate the
// unit vector, pick the Lloyd–Max cell of each coordinate, keys: residual,
// its norm and the signs of S r), laid out for the tensor cores:
//  * Rotation. With i = 16 p + q the Sylvester Hadamard matrix factors as
//    H_d = H_(d/16) (x) H_16, since popc(i & j) splits over the two bit
//    fields. One m16n8k16 MMA per 16-coordinate block applies H_16 (the
//    tile's 16 tokens are the rows; the fp16 inputs times +-1 are exact
//    products), then an in-register butterfly over the blocks applies
//    H_(d/16). The sign flip D is an XOR on the fp16 A operands.
//  * Norm from the rotated sums (Parseval: |H D x|^2 = d |x|^2), cells from
//    an fp32 search over the magnitude boundaries in registers (the codebooks
//    are antisymmetric by construction, the middle boundary is 0).
//  * Keys: r = y - c[idx] in fp32, z = S r on mma.sync with the fp16-exact S
//    and r split hi/lo (as in quantize_kernel).
//  * Exactness. fp32 decisions can differ from the fp64 path only next to a
//    boundary: any coordinate within TAU_Y of a compared boundary (or of 0),
//    and any key with |z_j| < TAU_Z, sends its vector to fixup_vector, which
//    redoes that vector in fp64 (the arithmetic of quantize_kernel, with z in
//    fp64 outright). TAU_Y is about 5x the worst fp32 error seen for the
//    rotated coordinates (rsqrt and the sums: ~2e-7), TAU_Z 10x the error of z.
//  * Packing. The C fragments of the rotation and of z hold, per lane, the
//    tokens g, g + 8 and coordinates 16 kk + 8 hs + 2 t + e, which are the key
//    codes and signs of this lane's own string (the layout of tq.h was made
//    for the attention kernel's A fragments). Value codes are transposed per
//    8 x 8 block with movmatrix. Each lane then stores its string with 64- or
//    128-bit coalesced stores.
// Partial tiles (an append that starts or ends inside a tile) keep the
// read-modify-write path of quantize_kernel.
#pragma once

namespace tq {
namespace {

constexpr float TAU_Y = 1.0e-6f;   // guard band of the fp32 cell decisions (rotated units)
constexpr float TAU_Z = 1.0e-5f;   // guard band of the fp32 QJL signs (units of r)

template <int D, int KB, int VB, int QJ>
struct FastQ {
    static constexpr bool OK = D <= 128 && KB <= 4 && VB <= 4;
    static constexpr int NB = D / 16;   // 16-coordinate blocks
};

// Cell search in registers for a B-bit antisymmetric codebook: H = 2^(B-1)
// non-negative levels, magnitude boundaries mb[k] = t[H + k], centroids
// cm[k] = c[H + k] (the middle boundary t[H - 1] is 0).
template <int B>
struct SymCells {
    static constexpr int H = 1 << (B - 1);
    float mb[H > 1 ? H - 1 : 1];
    float cm[H];
    __device__ __forceinline__ void load(const double* bounds, const double* cents)
    {
#pragma unroll
        for (int k = 0; k + 1 < H; ++k) mb[k] = (float)bounds[H + k];
#pragma unroll
        for (int k = 0; k < H; ++k) cm[k] = cents ? (float)cents[H + k] : 0.f;
    }
    // idx = #{j : y > t_j} (ties are within the guard band and go to fp64);
    // dacc = min(dacc, distances from y to every boundary the search compared,
    // 0 included); cen = c[idx] when CEN.
    template <bool CEN>
    __device__ __forceinline__ uint32_t encode(float y, float& dacc, float& cen) const
    {
        const float a = fabsf(y);
        uint32_t ip;   // H + m: the index of |y| among the non-negative cells
        float c = 0.f;
        if constexpr (B == 1) {
            ip = 1u;
            c = cm[0];
            dacc = fminf(dacc, a);
        } else if constexpr (B == 2) {
            const float d1 = a - mb[0];
            const bool c1 = d1 > 0.f;
            dacc = fminf(dacc, fminf(a, fabsf(d1)));
            ip = c1 ? 3u : 2u;
            if constexpr (CEN) c = c1 ? cm[1] : cm[0];
        } else if constexpr (B == 3) {
            const float d1 = a - mb[1];
            const bool c1 = d1 > 0.f;
            const float d2 = a - (c1 ? mb[2] : mb[0]);
            const bool c2 = d2 > 0.f;
            dacc = fminf(fminf(dacc, a), fminf(fabsf(d1), fabsf(d2)));
            ip = 4u + (c1 ? 2u : 0u) + (c2 ? 1u : 0u);
            if constexpr (CEN) c = c1 ? (c2 ? cm[3] : cm[2]) : (c2 ? cm[1] : cm[0]);
        } else {
            const float d1 = a - mb[3];
            const bool c1 = d1 > 0.f;
            const float d2 = a - (c1 ? mb[5] : mb[1]);
            const bool c2 = d2 > 0.f;
            const float d3 = a - (c1 ? (c2 ? mb[6] : mb[4]) : (c2 ? mb[2] : mb[0]));
            const bool c3 = d3 > 0.f;
            dacc = fminf(fminf(dacc, a), fminf(fabsf(d1), fminf(fabsf(d2), fabsf(d3))));
            ip = 8u + (c1 ? 4u : 0u) + (c2 ? 2u : 0u) + (c3 ? 1u : 0u);
            if constexpr (CEN)
                c = c1 ? (c2 ? (c3 ? cm[7] : cm[6]) : (c3 ? cm[5] : cm[4]))
                       : (c2 ? (c3 ? cm[3] : cm[2]) : (c3 ? cm[1] : cm[0]));
        }
        // y < 0: idx = H - 1 - m = (H + m) ^ (2H - 1)
        const uint32_t negm = (uint32_t)(__float_as_int(y) >> 31);
        if constexpr (CEN) cen = copysignf(c, y);
        return ip ^ (negm & (uint32_t)(2 * H - 1));
    }
};

// Per-warp scratch of the fp64 fix-up of one vector.
template <int D>
struct FixScratch {
    double r[D];        // fp64 residual (keys)
    uint8_t code[D];    // cells
    uint8_t sign[D];    // QJL signs (keys)
    uint8_t mark[D];    // QJL signs to recompute
    uint16_t norm, rho; // fp16 bits
};

// fp64 re-quantization of one fp16 vector by one warp (the arithmetic of
// quantize_kernel's first stage): cells, |x| and, for keys with QJL, the fp64
// residual r and rho, into fx. The signs are set by qjl_signs_* below.
template <int D, int B, bool KEY, int QJ>
__device__ __noinline__ void fixup_vector(const DevTables& tb, const __half* row, int lane,
                                          const double* bounds, const double* cents, FixScratch<D>& fx,
                                          unsigned& sat)
{
    constexpr int VPL = D / 32;
    double x[VPL];
    double ss = 0.0;
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
        x[k] = (double)__half2float(row[lane * VPL + k]);
        ss += x[k] * x[k];
        x[k] *= (double)tb.signs[lane * VPL + k];
    }
    ss = warp_sum(ss);
    wht_warp<VPL>(x, lane);
    const double nrm = sqrt(ss);
    const double scale = nrm > 0.0 ? (1.0 / sqrt((double)D)) / nrm : 0.0;
    double rr = 0.0;
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
        const double y = x[k] * scale;
        const int idx = encode_cell<B>(y, bounds);
        fx.code[lane * VPL + k] = (uint8_t)idx;
        if constexpr (KEY && QJ) {
            const double r = y - cents[idx];
            fx.r[lane * VPL + k] = r;
            rr += r * r;
        }
    }
    if constexpr (KEY && QJ) rr = warp_sum(rr);
    if (lane == 0) {
        fx.norm = norm_to_half_bits(nrm, sat);
        if constexpr (KEY && QJ) fx.rho = norm_to_half_bits(sqrt(rr), sat);
    }
    __syncwarp();
}

// Sign of z_j = S_j . r in fp64 (r = fx.r) for one sketch row j, by the warp.
template <int D>
__device__ __noinline__ void qjl_sign_one(const DevTables& tb, int lane, FixScratch<D>& fx, int j)
{
    double z = 0.0;
#pragma unroll
    for (int k = 0; k < D / 32; ++k) {
        const int i = lane + 32 * k;
        z += (double)__ldg(tb.s_t + (size_t)i * D + j) * fx.r[i];
    }
    z = warp_sum(z);
    if (lane == 0) fx.sign[j] = z >= 0.0 ? 1 : 0;
    __syncwarp();
}

// Signs of every z_j = S_j . r in fp64 (lane l takes rows l, l + 32, ...).
template <int D>
__device__ __noinline__ void qjl_signs_all(const DevTables& tb, int lane, FixScratch<D>& fx)
{
    constexpr int Q = D / 32;
    double z[Q];
#pragma unroll
    for (int q = 0; q < Q; ++q) z[q] = 0.0;
#pragma unroll 8
    for (int i = 0; i < D; ++i) {
        const double ri = fx.r[i];
#pragma unroll
        for (int q = 0; q < Q; ++q) z[q] += (double)__ldg(tb.s_t + (size_t)i * D + lane + 32 * q) * ri;
    }
#pragma unroll
    for (int q = 0; q < Q; ++q) fx.sign[lane + 32 * q] = z[q] >= 0.0 ? 1 : 0;
    __syncwarp();
}

// Set field [pos, pos + nb) of the lane string s (nb <= 8; the field may cross
// a word boundary) to v.
template <int NW>
__device__ __forceinline__ void put_bits(uint32_t (&s)[NW], int pos, uint32_t v, int nb)
{
    const int wi = pos >> 5, o = pos & 31;
    const uint32_t m = (1u << nb) - 1u;
    s[wi] = (s[wi] & ~(m << o)) | (v << o);
    if (o + nb > 32) s[wi + 1] = (s[wi + 1] & ~(m >> (32 - o))) | (v >> (32 - o));
}

template <int NW>
__device__ __forceinline__ uint32_t get_bits(const uint32_t (&s)[NW], int pos, int nb)
{
    const int wi = pos >> 5, o = pos & 31;
    uint32_t v = s[wi] >> o;
    if (o + nb > 32) v |= s[wi + 1] << (32 - o);
    return v & ((1u << nb) - 1u);
}

// (a, b) <- (a + b, a - b) on two fp32 pairs at once (f32x2 add and sub).
__device__ __forceinline__ void butterfly2(float& a0, float& a1, float& b0, float& b1)
{
    asm("{\n .reg .b64 A, B, S, T;\n"
        " mov.b64 A, {%0, %1};\n mov.b64 B, {%2, %3};\n"
        " add.rn.f32x2 S, A, B;\n sub.rn.f32x2 T, A, B;\n"
        " mov.b64 {%0, %1}, S;\n mov.b64 {%2, %3}, T;\n}\n"
        : "+f"(a0), "+f"(a1), "+f"(b0), "+f"(b1));
}

// Shared memory of one warp of quantize_fast: the rotated values of one matrix
// (or the key residuals), element c of C fragment [kk][hs] at y[2 kk + hs][lane].c,
// and the cells, byte c of code[m][2 kk + hs][lane] (m = 0 keys, 1 values).
template <int D>
struct QWarp {
    float4 y[D / 8][32];
    uint32_t code[2][D / 8][32];
    FixScratch<D> fx;
};

template <int D>
struct QFastSmem {
    QWarp<D> w[4];
    uint32_t sgt[256];              // sign scatter: the 8 sign bits of n-tiles 2 kk, 2 kk + 1 -> word bits
    uint32_t dmask[D / 2];          // fp16x2 sign-flip masks of coordinate pairs
    double tk[16], tv[16], ck[16];  // boundaries and key centroids (fp64 copies of the fp32 tables)
};

template <int D, int KB, int VB, int QJ>
__global__ void __launch_bounds__(128) quantize_fast(DevTables tb, QuantizeArgs a)
{
    using Tr = QuantTraits<D, KB, VB, QJ>;
    using Lay = TileLayout<D, KB, VB, QJ>;
    constexpr int NB = FastQ<D, KB, VB, QJ>::NB, NW = Tr::SBYTES / 4, NI = D / 8;
    extern __shared__ __align__(16) unsigned char qf_smem_raw[];
    QFastSmem<D>& sm = *reinterpret_cast<QFastSmem<D>*>(qf_smem_raw);

    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
    const int b = blockIdx.z, h = blockIdx.y;
    for (int i = tid; i < D / 2; i += 128)
        sm.dmask[i] = (tb.signs[2 * i] < 0.f ? 0x8000u : 0u) | (tb.signs[2 * i + 1] < 0.f ? 0x80000000u : 0u);
    if (tid < (1 << KB) - 1) sm.tk[tid] = tb.bounds_k[tid];
    if (tid < (1 << VB) - 1) sm.tv[tid] = tb.bounds_v[tid];
    if (tid < (1 << KB)) sm.ck[tid] = tb.centroids_kd[tid];
    if constexpr (QJ) {
        // source bit 4 hs + 2 rw + e (n-tile 2 kk + hs, element 2 rw + e) is the sign
        // of pair 4 kk + 2 hs + rw, element e: byte fields put it at bit
        // 6 + rw + 8 hs + 16 e of word kk (of the key words for (3, 4, 1), of the
        // value words for (2, 3, 1)), sign words at 16 e + 2 hs + rw (+ 4 (kk & 3))
        for (int x = tid; x < 256; x += 128) {
            uint32_t v = 0u;
#pragma unroll
            for (int bsrc = 0; bsrc < 8; ++bsrc) {
                if (!((x >> bsrc) & 1)) continue;
                const int hs = bsrc >> 2, rw = (bsrc >> 1) & 1, e = bsrc & 1;
                using L = TileLayout<D, KB, VB, QJ>;
                v |= 1u << (L::KS_BYTES || L::VS_BYTES ? 6 + rw + 8 * hs + 16 * e : 16 * e + 2 * hs + rw);
            }
            sm.sgt[x] = v;
        }
    }
    __syncthreads();

    const int start = a.start_pos[b];
    if (start < 0 || (long long)start + a.T > (long long)a.capacity) return;   // quantize_kernel flags it
    const int tile = start / 16 + blockIdx.x * 4 + w;
    const int first = tile * 16;
    if (first < start || first + 16 > start + a.T) return;   // partial or past the end: quantize_kernel
    const size_t row0 = (((size_t)b * a.Hkv + h) * (size_t)a.T + (size_t)(first - start)) * D;
    QWarp<D>& qw = sm.w[w];

    SymCells<KB> kcells;
    SymCells<VB> vcells;
    kcells.load(sm.tk, QJ ? sm.ck : nullptr);
    vcells.load(sm.tv, nullptr);

    // H_16 as B fragments (+-1 fp16): b0 rows 2t, 2t+1, b1 rows 8 + 2t, 9 + 2t; column 8 hs + g
    uint32_t hb[2][2];
#pragma unroll
    for (int hs = 0; hs < 2; ++hs) {
        const int col = 8 * hs + g;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const int r0 = 8 * q + 2 * t;
            const uint32_t lo = (__popc(r0 & col) & 1) ? 0xBC00u : 0x3C00u;
            const uint32_t hi = (__popc((r0 + 1) & col) & 1) ? 0xBC00u : 0x3C00u;
            hb[hs][q] = lo | (hi << 16);
        }
    }

    // Rotated unit vectors of one matrix of the tile into qw.y (element c of
    // [kk][hs]: token g + 8 (c >> 1), coordinate 16 kk + 8 hs + 2t + (c & 1)),
    // and the fp16 norms of the rows g, g + 8.
    unsigned sat = 0u;
    auto rotate = [&](const __half* X, uint16_t (&nrm)[2]) {
        const uint32_t* rg = reinterpret_cast<const uint32_t*>(X + row0 + (size_t)g * D);
        const uint32_t* rh = reinterpret_cast<const uint32_t*>(X + row0 + (size_t)(g + 8) * D);
        uint32_t av[NB][4];
#pragma unroll
        for (int p = 0; p < NB; ++p) {
            av[p][0] = __ldg(rg + 8 * p + t);
            av[p][1] = __ldg(rh + 8 * p + t);
            av[p][2] = __ldg(rg + 8 * p + 4 + t);
            av[p][3] = __ldg(rh + 8 * p + 4 + t);
        }
        float y[NB][2][4];
#pragma unroll
        for (int p = 0; p < NB; ++p) {
            const uint32_t m0 = sm.dmask[8 * p + t], m1 = sm.dmask[8 * p + 4 + t];
            const uint32_t a0 = av[p][0] ^ m0, a1 = av[p][1] ^ m0, a2 = av[p][2] ^ m1, a3 = av[p][3] ^ m1;
#pragma unroll
            for (int hs = 0; hs < 2; ++hs) mma_16816_first(y[p][hs], a0, a1, a2, a3, hb[hs][0], hb[hs][1]);
        }
        // H_(d/16) over the blocks
#pragma unroll
        for (int st = 1; st < NB; st <<= 1) {
#pragma unroll
            for (int p = 0; p < NB; ++p) {
                if (p & st) continue;
#pragma unroll
                for (int hs = 0; hs < 2; ++hs) {
                    butterfly2(y[p][hs][0], y[p][hs][1], y[p + st][hs][0], y[p + st][hs][1]);
                    butterfly2(y[p][hs][2], y[p][hs][3], y[p + st][hs][2], y[p + st][hs][3]);
                }
            }
        }
        float ssg = 0.f, ssh = 0.f;
#pragma unroll
        for (int p = 0; p < NB; ++p) {
#pragma unroll
            for (int hs = 0; hs < 2; ++hs) {
                ssg = fmaf(y[p][hs][0], y[p][hs][0], fmaf(y[p][hs][1], y[p][hs][1], ssg));
                ssh = fmaf(y[p][hs][2], y[p][hs][2], fmaf(y[p][hs][3], y[p][hs][3], ssh));
            }
        }
#pragma unroll
        for (int o = 1; o <= 2; o <<= 1) {
            ssg += __shfl_xor_sync(kFull, ssg, o);
            ssh += __shfl_xor_sync(kFull, ssh, o);
        }
        // |x| = sqrt(ss / d); y / (sqrt(d) |x|) = y / sqrt(ss)
        nrm[0] = norm_to_half_bits((double)sqrtf(ssg * (1.0f / (float)D)), sat);
        nrm[1] = norm_to_half_bits((double)sqrtf(ssh * (1.0f / (float)D)), sat);
        const float sg = ssg > 0.f ? rsqrtf(ssg) : 0.f, sh = ssh > 0.f ? rsqrtf(ssh) : 0.f;
#pragma unroll
        for (int p = 0; p < NB; ++p) {
#pragma unroll
            for (int hs = 0; hs < 2; ++hs)
                qw.y[2 * p + hs][lane] = make_float4(y[p][hs][0] * sg, y[p][hs][1] * sg, y[p][hs][2] * sh,
                                                     y[p][hs][3] * sh);
        }
        __syncwarp();
    };

    uint16_t kn[2], rn[2] = {0, 0}, vn[2];   // fp16 norms of the rows g, g + 8
    bool fixk[2] = {false, false}, fixv[2] = {false, false};
    // QJL signs and close calls: bit 4 nt + c (n-tile nt, element c)
    unsigned long long sgn = 0ull, zcl = 0ull;
    {
        // ---------------- keys: cells (and residuals in place of y)
        rotate(a.k, kn);
        float rr[2] = {0.f, 0.f}, dk[2] = {1.f, 1.f};
#pragma unroll 1
        for (int i = 0; i < NI; ++i) {
            float4 v = qw.y[i][lane];
            float yy[4] = {v.x, v.y, v.z, v.w};
            uint32_t idx[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float cen;
                idx[c] = kcells.template encode<QJ != 0>(yy[c], dk[c >> 1], cen);
                if constexpr (QJ) {
                    yy[c] -= cen;
                    rr[c >> 1] = fmaf(yy[c], yy[c], rr[c >> 1]);
                }
            }
            qw.code[0][i][lane] = __byte_perm(__byte_perm(idx[0], idx[1], 0x0040u), __byte_perm(idx[2], idx[3], 0x0040u), 0x5410u);
            if constexpr (QJ) qw.y[i][lane] = make_float4(yy[0], yy[1], yy[2], yy[3]);
        }
        fixk[0] = dk[0] < TAU_Y;
        fixk[1] = dk[1] < TAU_Y;
        if constexpr (QJ) {
#pragma unroll
            for (int o = 1; o <= 2; o <<= 1) {
                rr[0] += __shfl_xor_sync(kFull, rr[0], o);
                rr[1] += __shfl_xor_sync(kFull, rr[1], o);
            }
#pragma unroll
            for (int rw = 0; rw < 2; ++rw) rn[rw] = norm_to_half_bits((double)sqrtf(rr[rw]), sat);
            __syncwarp();
            // z = S r: A = 2^12 r as hi + lo fp16 (k-step kk: coordinates 16 kk + ...;
            // A rows: q = 0 token g coords 2t.., 1 token g + 8, 2 token g coords 8 + 2t.., 3 token g + 8)
            uint32_t ah[NB][4], al[NB][4];
#pragma unroll
            for (int kk = 0; kk < NB; ++kk) {
#pragma unroll
                for (int hs = 0; hs < 2; ++hs) {
                    const float4 r = qw.y[2 * kk + hs][lane];
                    const float s0 = r.x * 4096.f, s1 = r.y * 4096.f, s2 = r.z * 4096.f, s3 = r.w * 4096.f;
                    const __half2 h01 = __floats2half2_rn(s0, s1), h23 = __floats2half2_rn(s2, s3);
                    const float2 f01 = __half22float2(h01), f23 = __half22float2(h23);
                    ah[kk][2 * hs] = *reinterpret_cast<const uint32_t*>(&h01);
                    ah[kk][2 * hs + 1] = *reinterpret_cast<const uint32_t*>(&h23);
                    al[kk][2 * hs] = pack_half2(s0 - f01.x, s1 - f01.y);
                    al[kk][2 * hs + 1] = pack_half2(s2 - f23.x, s3 - f23.y);
                }
            }
            const float thr = TAU_Z * 4096.f;
            // S^T fragments of n-tile nt + 1 load while nt multiplies
            uint2 bfn[NB];
#pragma unroll
            for (int kk = 0; kk < NB; ++kk) bfn[kk] = __ldg(tb.s_frag + (size_t)kk * (D / 8) * 32 + lane);
#pragma unroll 1
            for (int nt = 0; nt < D / 8; ++nt) {
                uint2 bf[NB];
#pragma unroll
                for (int kk = 0; kk < NB; ++kk) bf[kk] = bfn[kk];
                if (nt + 1 < D / 8) {
#pragma unroll
                    for (int kk = 0; kk < NB; ++kk)
                        bfn[kk] = __ldg(tb.s_frag + ((size_t)kk * (D / 8) + nt + 1) * 32 + lane);
                }
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int kk = 0; kk < NB; ++kk) {
                    mma_16816(acc, ah[kk][0], ah[kk][1], ah[kk][2], ah[kk][3], bf[kk].x, bf[kk].y);
                    mma_16816(acc, al[kk][0], al[kk][1], al[kk][2], al[kk][3], bf[kk].x, bf[kk].y);
                }
                // sign bits: the complemented float sign bits (z >= 0 -> 1; -0 counts as 0,
                // and |z| = 0 is a close call anyway)
                const uint32_t bits =
                    (~((__float_as_uint(acc[0]) >> 31) | ((__float_as_uint(acc[1]) >> 30) & 2u) |
                       ((__float_as_uint(acc[2]) >> 29) & 4u) | ((__float_as_uint(acc[3]) >> 28) & 8u))) & 15u;
                sgn |= (unsigned long long)bits << (4 * nt);
                if (fminf(fminf(fabsf(acc[0]), fabsf(acc[1])), fminf(fabsf(acc[2]), fabsf(acc[3]))) < thr) {
                    uint32_t close = 0u;
#pragma unroll
                    for (int c = 0; c < 4; ++c) close |= (fabsf(acc[c]) < thr ? 1u : 0u) << c;
                    zcl |= (unsigned long long)close << (4 * nt);
                }
            }
            // rows with a close call (elements 0, 1: token g; 2, 3: token g + 8)
            fixk[0] |= (zcl & 0x3333333333333333ull) != 0ull;
            fixk[1] |= (zcl & 0xCCCCCCCCCCCCCCCCull) != 0ull;
        }
    }
    {
        // ---------------- values: cells
        rotate(a.v, vn);
        float dv[2] = {1.f, 1.f};
#pragma unroll 1
        for (int i = 0; i < NI; ++i) {
            const float4 v = qw.y[i][lane];
            const float yy[4] = {v.x, v.y, v.z, v.w};
            uint32_t idx[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float cen;
                idx[c] = vcells.template encode<false>(yy[c], dv[c >> 1], cen);
            }
            qw.code[1][i][lane] = __byte_perm(__byte_perm(idx[0], idx[1], 0x0040u), __byte_perm(idx[2], idx[3], 0x0040u), 0x5410u);
        }
        fixv[0] = dv[0] < TAU_Y;
        fixv[1] = dv[1] < TAU_Y;
    }
    __syncwarp();

    // ---------------- fp64 fix-ups (rare): every token a lane flagged
    {
        FixScratch<D>& fx = qw.fx;
        const uint32_t bk0 = __ballot_sync(kFull, fixk[0]), bk1 = __ballot_sync(kFull, fixk[1]);
        const uint32_t bv0 = __ballot_sync(kFull, fixv[0]), bv1 = __ballot_sync(kFull, fixv[1]);
        // token n (0..15) is flagged when any of its four lanes is
        auto tokens = [](uint32_t b0, uint32_t b1) {
            uint32_t m = 0u;
#pragma unroll
            for (int gg = 0; gg < 8; ++gg) {
                if ((b0 >> (4 * gg)) & 0xFu) m |= 1u << gg;
                if ((b1 >> (4 * gg)) & 0xFu) m |= 1u << (gg + 8);
            }
            return m;
        };
        uint32_t fk = tokens(bk0, bk1), fv = tokens(bv0, bv1);
#pragma unroll 1
        for (int kind = 0; kind < 2; ++kind) {
            uint32_t f = kind == 0 ? fk : fv;
            while (f) {
                const int n = __ffs(f) - 1, rw = n >> 3;
                f &= f - 1;
                const bool own = g == (n & 7);
                if (kind == 0)
                    fixup_vector<D, KB, true, QJ>(tb, a.k + row0 + (size_t)n * D, lane, sm.tk, sm.ck, fx, sat);
                else
                    fixup_vector<D, VB, false, 0>(tb, a.v + row0 + (size_t)n * D, lane, sm.tv, nullptr, fx, sat);
                if (QJ && kind == 0) {
                    // Unchanged cells: r moved by rounding only, so only the signs whose
                    // fp32 z was within TAU_Z are redone. Changed cells: all of them.
                    bool diff = false;
                    if (own) {
#pragma unroll 1
                        for (int i = 0; i < NI; ++i) {
                            const uint32_t word = qw.code[0][i][lane];
                            const int kk = i >> 1, hs = i & 1, nt = i;   // n-tile 2 kk + hs = i
#pragma unroll
                            for (int e = 0; e < 2; ++e) {
                                const int c = 2 * rw + e, j = 16 * kk + 8 * hs + 2 * t + e;
                                diff |= ((word >> (8 * c)) & 0xFFu) != fx.code[j];
                                fx.sign[j] = (uint8_t)((sgn >> (4 * nt + c)) & 1ull);
                                fx.mark[j] = (uint8_t)((zcl >> (4 * nt + c)) & 1ull);
                            }
                        }
                    }
                    if (__any_sync(kFull, diff)) {
                        qjl_signs_all<D>(tb, lane, fx);
                    } else {
                        __syncwarp();
#pragma unroll 1
                        for (int q = 0; q < D / 32; ++q) {
                            uint32_t m = __ballot_sync(kFull, fx.mark[lane + 32 * q] != 0);
                            while (m) {
                                const int j = 32 * q + __ffs(m) - 1;
                                m &= m - 1;
                                qjl_sign_one<D>(tb, lane, fx, j);
                            }
                        }
                    }
                }
                if (own) {
#pragma unroll 1
                    for (int i = 0; i < NI; ++i) {
                        uint32_t word = qw.code[kind][i][lane];
                        const int kk = i >> 1, hs = i & 1;
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int c = 2 * rw + e, j = 16 * kk + 8 * hs + 2 * t + e;
                            word = (word & ~(0xFFu << (8 * c))) | ((uint32_t)fx.code[j] << (8 * c));
                            if (QJ && kind == 0) {
                                const int bit = 4 * i + c;
                                sgn = (sgn & ~(1ull << bit)) | ((unsigned long long)fx.sign[j] << bit);
                            }
                        }
                        qw.code[kind][i][lane] = word;
                    }
                    if (kind == 0) {
                        kn[rw] = fx.norm;
                        if constexpr (QJ) rn[rw] = fx.rho;
                    } else {
                        vn[rw] = fx.norm;
                    }
                }
                __syncwarp();
            }
        }
    }

    // ---------------- the lane string
    // Key pair 4 kk + r: token g + 8 (r & 1) at coordinates 16 kk + 8 (r >> 1) + 2t + e,
    // element c = 2 (r & 1) + e of [kk][hs = r >> 1]; its signs: n-tile 2 kk + hs.
    // Fields never overlap and s starts at 0, so every field is OR-ed in.
    using LayT = TileLayout<D, KB, VB, QJ>;
    constexpr bool KBYTE = LayT::KS_BYTES || KB == 4;       // key pair p = byte p
    uint32_t s[NW];
#pragma unroll
    for (int i = 0; i < NW; ++i) s[i] = 0u;
    auto put_or = [&](int pos, uint32_t v, int nb) {
        const int wi = pos >> 5, o = pos & 31;
        s[wi] |= v << o;
        if (o + nb > 32) s[wi + 1] |= v >> (32 - o);
    };
    constexpr uint32_t VM = (1u << VB) - 1u;
#pragma unroll
    for (int kk = 0; kk < NB; ++kk) {
        const uint32_t kw0 = qw.code[0][2 * kk][lane], kw1 = qw.code[0][2 * kk + 1][lane];
        const uint32_t vw0 = qw.code[1][2 * kk][lane], vw1 = qw.code[1][2 * kk + 1][lane];
        // byte r = 2 hs + rw of lo / hi: the pair's element 0 / 1
        const uint32_t lo = __byte_perm(kw0, kw1, 0x6420u), hi = __byte_perm(kw0, kw1, 0x7531u);
        const uint32_t pairs = lo | (hi << KB);                 // byte r: the pair's KB-bit fields
        if constexpr (KBYTE) {
            s[kk] |= pairs;                                     // word kk = pairs 4 kk .. 4 kk + 3
        } else if constexpr (KB == 2) {
            const uint32_t t4 = pairs | (pairs >> 4);           // nibble fields
            put_or(16 * kk, __byte_perm(t4, 0u, 0x4420u) & 0xFFFFu, 16);
        } else if constexpr (KB == 1) {
            const uint32_t t2 = pairs | (pairs >> 6);
            const uint32_t u = __byte_perm(t2, 0u, 0x4420u) & 0xFFFFu;
            put_or(8 * kk, (u | (u >> 4)) & 0xFFu, 8);
        } else {
#pragma unroll
            for (int r = 0; r < 4; ++r) put_or(LayT::kbit(4 * kk + r, 0), (pairs >> (8 * r)) & 0xFFu, 2 * KB);
        }
        if constexpr (QJ) {
            const uint32_t sb = (uint32_t)(sgn >> (8 * kk)) & 0xFFu;
            const uint32_t m = sm.sgt[sb];
            if constexpr (LayT::KS_BYTES)
                s[kk] |= m;
            else if constexpr (LayT::VS_BYTES)
                s[LayT::VB0 / 32 + kk] |= m;
            else
                s[LayT::SB0 / 32 + (kk >> 2)] |= m << (4 * (kk & 3));
        }
        // values: transpose the 8 x 8 blocks (tokens x coordinates); before, lane
        // (g, t) holds token g + 8 half at coordinates 2t, 2t + 1; after, tokens
        // 2t, 2t + 1 (+ 8 half) at coordinate g: value pair j = 2 half + hs
#pragma unroll
        for (int hs = 0; hs < 2; ++hs) {
            const uint32_t vw = hs ? vw1 : vw0;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const uint32_t x = ((vw >> (16 * half)) & 0xFFu) | (((vw >> (16 * half + 8)) & 0xFFu) << 16);
                const int p = 4 * kk + 2 * half + hs;
                if constexpr (VB == 4) {
                    // odd tokens shifted by 4 before the transposition: the pair's byte
                    // is then the OR of the two halves
                    const uint32_t tr = movmatrix_trans(x << (4 * (g & 1)));
                    put_or(LayT::vbit(p, 0), (tr | (tr >> 16)) & 0xFFu, 8);
                } else {
                    const uint32_t tr = movmatrix_trans(x);
                    put_or(LayT::vbit(p, 0), tr & VM, VB);
                    put_or(LayT::vbit(p, 1), (tr >> 16) & VM, VB);
                }
            }
        }
    }

    uint8_t* tp = a.cache + (((size_t)b * a.Hkv + h) * (size_t)(a.capacity / 16) + tile) * (size_t)a.tile_bytes;
#pragma unroll
    for (int c = 0; c < Tr::NCH; ++c) {
        uint8_t* dst = tp + ((size_t)c * 32 + lane) * Tr::CB;
        if constexpr (Tr::CW == 4)
            *reinterpret_cast<uint4*>(dst) = make_uint4(s[4 * c], s[4 * c + 1], s[4 * c + 2], s[4 * c + 3]);
        else if constexpr (Tr::CW == 2)
            *reinterpret_cast<uint2*>(dst) = make_uint2(s[2 * c], s[2 * c + 1]);
        else
            *reinterpret_cast<uint32_t*>(dst) = s[c];
    }
    if (t == 0) {
        uint8_t* nb = tp + Tr::CODE_BYTES;
        if constexpr (QJ)
            *reinterpret_cast<uint2*>(nb + 8 * g) =
                make_uint2((uint32_t)kn[0] | ((uint32_t)rn[0] << 16), (uint32_t)kn[1] | ((uint32_t)rn[1] << 16));
        else
            *reinterpret_cast<uint32_t*>(nb + 4 * g) = (uint32_t)kn[0] | ((uint32_t)kn[1] << 16);
        *reinterpret_cast<uint32_t*>(nb + Tr::KNB + 4 * g) = (uint32_t)vn[0] | ((uint32_t)vn[1] << 16);
    }
    if (sat) atomicOr(tb.status, TQ_STATUS_NORM_SAT);
}

}  // namespace
}  // namespace tq
