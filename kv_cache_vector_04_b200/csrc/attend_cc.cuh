// CUDA-core variant of the split kernel (tq_attend_cudacore): the arithmetic
// the plan of the pages sets out for tq_attend, kept beside the tensor-core
// kernel as a measured comparison. Logits come from a query x centroid lookup
// table in shared memory, the QJL term from sign-nibble tables (mode 1) or from
// bit-plane popcounts (mode 2), and P V runs as CUDA-core FMAs; the query
// prologue, the stream-K split of the tiles and the reduce are the tensor-core
// path's own, so the two kernels read the same bytes and write the same
// partials. Built for TurboQuant at 4 bits with d = 128, the format of the
// Llama-3.3-70B-shaped workload.
//
// Included by attend_impl.cuh inside its namespace, after the split kernel's
// helpers.
#pragma once

struct CcTraits {
    static constexpr int D = 128, KB = 3, VB = 4, QJ = 1;
    using Tr = AttTraits<D, KB, VB, QJ>;
    static constexpr int WARPS = 16, NT = 32 * WARPS, KK = D / 16;
    static constexpr int TB = Tr::TILE_BYTES;
    static constexpr int RS = D + 2;                           // merge-buffer row
    static constexpr size_t TK = (size_t)D * 8 * 8 * 4;          // [coordinate][code][head] fp32
    static constexpr size_t QT = (size_t)4 * KK * 16 * 8 * 4;    // [t][kk][nibble or plane][head]
    static constexpr size_t RING = (size_t)WARPS * 2 * TB;       // two tile slots a warp
    static constexpr size_t MERGE = (size_t)WARPS * 8 * RS * 4;  // aliases the ring after a segment
    static constexpr size_t BODY = RING > MERGE ? RING : MERGE;
    static constexpr size_t WV = (size_t)WARPS * 16 * 8 * 4;     // p |v| of a tile, per warp
    static constexpr size_t QS = (size_t)8 * D * 4;              // q~ of the unit, fp32
    static constexpr size_t NS = (size_t)8 * D * 4;              // QJL fixed-point codes n
    static constexpr size_t OFF_QT = TK, OFF_BODY = OFF_QT + QT, OFF_WV = OFF_BODY + BODY;
    static constexpr size_t OFF_QS = OFF_WV + WV, OFF_NS = OFF_QS + QS, OFF_TAB = OFF_NS + NS;
    static constexpr size_t SMEM = OFF_TAB + 64 * 4;             // + value table, u, T
    static_assert(SMEM <= Tr::SMEM_CAP, "CUDA-core split CTA exceeds shared memory");
    static_assert(TB % 16 == 0 && OFF_BODY % 16 == 0, "bulk copies need 16-byte sizes and addresses");
};

// Word kk (0..15) of lane l's string in a tile image (16-byte chunks, chunk-major).
__device__ __forceinline__ const uint32_t* cc_word(const uint8_t* tile, int l, int kk)
{
    return reinterpret_cast<const uint32_t*>(tile + ((kk >> 2) * 32 + l) * 16 + (kk & 3) * 4);
}

template <int MODE>
__global__ void __launch_bounds__(CcTraits::NT, 1) attend_cc(DevTables tb, AttendArgs a)
{
    using C = CcTraits;
    constexpr int D = C::D, KK = C::KK, WARPS = C::WARPS, NT = C::NT, TB = C::TB, RS = C::RS;
    __shared__ __align__(8) uint64_t bars[WARPS * 2];
    extern __shared__ uint4 dyn_smem[];
    uint8_t* sm = reinterpret_cast<uint8_t*>(dyn_smem);
    float* tk = reinterpret_cast<float*>(sm);                         // [i][code][h]
    float* qt = reinterpret_cast<float*>(sm + C::OFF_QT);             // mode 1: [t][kk][nibble][h]
    uint32_t* pw = reinterpret_cast<uint32_t*>(sm + C::OFF_QT);       // mode 2: [t][kk][plane][h]
    uint8_t* ring = sm + C::OFF_BODY;
    float* mrg = reinterpret_cast<float*>(sm + C::OFF_BODY);
    float* wv = reinterpret_cast<float*>(sm + C::OFF_WV);             // [warp][token][h]
    float* qs = reinterpret_cast<float*>(sm + C::OFF_QS);             // [h][i]
    int* ns = reinterpret_cast<int*>(sm + C::OFF_NS);                 // [h][j]
    float* vtab = reinterpret_cast<float*>(sm + C::OFF_TAB);          // [16] value levels
    float* uq = vtab + 16;                                            // [8] QJL scale u per head
    int* tq = reinterpret_cast<int*>(vtab + 24);                      // [8] T = sum of n per head
    float* ktab = vtab + 32;                                          // [8] key levels

    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int tau = lane >> 1, hh = lane & 1;                          // logits: token, head half
    const int g = tau & 7, rho = tau >> 3;
    const int c = blockIdx.x;
    const long long G = gridDim.x;
    const int groups = a.plan.groups, upb = a.Hkv * groups;
    if (tid < 16) vtab[tid] = __low2float(*reinterpret_cast<const __half2*>(tb.lut_v + tid));
    else if (tid < 24) ktab[tid - 16] = __low2float(*reinterpret_cast<const __half2*>(tb.lut_k + (tid - 16)));
    uint8_t* wring = ring + (size_t)w * 2 * TB;
    const uint32_t ring_s = (uint32_t)__cvta_generic_to_shared(wring);
    const uint32_t bar_s = (uint32_t)__cvta_generic_to_shared(bars + w * 2);
    if (lane == 0) {
        mbar_init(bar_s, 1);
        mbar_init(bar_s + 8, 1);
        fence_mbar_init();
    }
    __syncwarp();
    pdl_trigger();
    pdl_wait();
    const long long W = a.prefix[a.B];
    const long long x0 = (long long)c * W / G, x1 = (long long)(c + 1) * W / G;
    if (x0 >= x1) return;
    const int lim = min(a.max_len, a.capacity);
    uint32_t issued = 0, consumed = 0;
    bool stalled = false;

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

        // ---- the unit's tables: q~ and n back from the prologue's fragments
        {
            const uint4* fr = reinterpret_cast<const uint4*>(a.qfrag) + u * KK * 64;
            if (tid < KK * 32) {                     // codebook B: head col, coordinates c0 + {0, 1, 8, 9}
                const int kk = tid >> 5, col = (tid >> 2) & 7, t = tid & 3, c0 = 16 * kk + 2 * t;
                const uint4 v = fr[kk * 64 + col * 4 + t];
                const float2 h01 = __half22float2(*reinterpret_cast<const __half2*>(&v.x));
                const float2 h89 = __half22float2(*reinterpret_cast<const __half2*>(&v.y));
                const float2 l01 = __half22float2(*reinterpret_cast<const __half2*>(&v.z));
                const float2 l89 = __half22float2(*reinterpret_cast<const __half2*>(&v.w));
                qs[col * D + c0] = h01.x + l01.x;
                qs[col * D + c0 + 1] = h01.y + l01.y;
                qs[col * D + c0 + 8] = h89.x + l89.x;
                qs[col * D + c0 + 9] = h89.y + l89.y;
            } else if (tid < KK * 32 + (D / 32) * 32) {   // QJL B: head hc, 8 coordinates
                const int e = tid - KK * 32, J = e >> 5, ln = e & 31, hc = ln >> 2, tt = ln & 3;
                const uint4 v = fr[J * 64 + 32 + ln];
                const uint32_t bh[2] = {v.x, v.y}, bl[2] = {v.z, v.w};
#pragma unroll
                for (int half = 0; half < 2; ++half)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int n = (int)(int8_t)(bh[half] >> (8 * i)) * 256 + (int)((bl[half] >> (8 * i)) & 0xFFu);
                        ns[hc * D + qjl_dim<2>(J, tt, half, i)] = n;
                    }
            } else if (tid < KK * 32 + (D / 32) * 32 + 8) {   // u of head h (2 u / 64 in the constants)
                const int h = tid - KK * 32 - (D / 32) * 32;
                const uint4 v = fr[(D / 32) * 64 + 32 + (h >> 1)];
                uq[h] = __uint_as_float((h & 1) ? v.y : v.x) * 32.f;
            }
        }
        __syncthreads();
        if (w < 8) {   // T of head w
            int s = 0;
            for (int i = lane; i < D; i += 32) s += ns[w * D + i];
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) s += __shfl_xor_sync(kFull, s, o);
            if (lane == 0) tq[w] = s;
        }
        for (int e = tid; e < D * 8 * 8; e += NT) {   // q~_h[i] x level[code]
            const int h = e & 7, code = (e >> 3) & 7, i = e >> 6;
            tk[e] = qs[h * D + i] * ktab[code];
        }
        for (int e = tid; e < 4 * KK * 16 * 8; e += NT) {
            // nibble (mode 1) or plane (mode 2) q of word (t, kk), head h; its four
            // projection rows: 16 kk + 2t, + 8, + 1, + 9
            const int h = e & 7, q = (e >> 3) & 15, kk = (e >> 7) & 7, t = e >> 10;
            const int R[4] = {16 * kk + 2 * t, 16 * kk + 8 + 2 * t, 16 * kk + 2 * t + 1, 16 * kk + 9 + 2 * t};
            if constexpr (MODE == 1) {
                float s = 0.f;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float xv = uq[h] * (float)ns[h * D + R[k]];
                    s += ((q >> k) & 1) ? xv : -xv;
                }
                qt[e] = s;
            } else {
                uint32_t v = 0;
#pragma unroll
                for (int k = 0; k < 4; ++k) v |= (((uint32_t)ns[h * D + R[k]] >> q) & 1u) << (6 + 8 * k);
                pw[e] = v;
            }
        }
        __syncthreads();

        float m[4], l[4], acc[4][8];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            m[k] = -CUDART_INF_F;
            l[k] = 0.f;
        }
#pragma unroll
        for (int mm = 0; mm < 4; ++mm)
#pragma unroll
            for (int h = 0; h < 8; ++h) acc[mm][h] = 0.f;

        const uint8_t* sbase = a.cache + ((size_t)b * a.Hkv + hkv) * (size_t)(a.capacity >> 4) * (size_t)a.tile_bytes;
        const int ntile = se - sb;
        fence_proxy_async();
        if (!stalled && w < ntile) {
            if (lane == 0) bulk_load(ring_s + (issued & 1u) * TB, sbase + (size_t)(sb + w) * TB, TB, bar_s + 8 * (issued & 1u));
            ++issued;
        }
        float* wvw = wv + w * 128;
#pragma unroll 1
        for (int p = w; p < ntile && !stalled; p += WARPS) {
            if (p + WARPS < ntile) {
                fence_proxy_async();
                if (lane == 0)
                    bulk_load(ring_s + (issued & 1u) * TB, sbase + (size_t)(sb + p + WARPS) * TB, TB,
                              bar_s + 8 * (issued & 1u));
                ++issued;
            }
            const uint32_t slot = consumed & 1u;
            if (!mbar_wait(bar_s + 8 * slot, (consumed >> 1) & 1u)) {
                stalled = true;
                if (lane == 0) atomicOr(tb.status, TQ_STATUS_WAIT_TIMEOUT);
                break;
            }
            ++consumed;
            const uint8_t* tile = wring + slot * TB;
            const int tl = sb + p;

            // ---- logits of token tau for heads 4 hh .. 4 hh + 3
            float cb[4] = {0.f, 0.f, 0.f, 0.f}, qj[4] = {0.f, 0.f, 0.f, 0.f};
            int iq[4] = {0, 0, 0, 0};
#pragma unroll 1
            for (int t = 0; t < 4; ++t) {
                const uint4 w0 = *reinterpret_cast<const uint4*>(cc_word(tile, 4 * g + t, 0));
                const uint4 w1 = *reinterpret_cast<const uint4*>(cc_word(tile, 4 * g + t, 4));
                const uint32_t kw[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
                for (int kk = 0; kk < KK; ++kk) {
                    const uint32_t word = kw[kk];
#pragma unroll
                    for (int r2 = 0; r2 < 2; ++r2) {          // byte rho + 2 r2: coordinates 16 kk + 8 r2 + 2t + e
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int code = (word >> (8 * (rho + 2 * r2) + 3 * e)) & 7;
                            const int i = 16 * kk + 8 * r2 + 2 * t + e;
                            const float4 v = *reinterpret_cast<const float4*>(tk + ((i * 8 + code) * 8 + 4 * hh));
                            cb[0] += v.x;
                            cb[1] += v.y;
                            cb[2] += v.z;
                            cb[3] += v.w;
                        }
                    }
                    if constexpr (MODE == 1) {
                        const uint32_t sx = (word >> (6 + rho)) & 0x01010101u;
                        const int nib = (int)(((sx * 0x204081u) >> 21) & 15u);
                        const float4 v = *reinterpret_cast<const float4*>(qt + (((t * KK + kk) * 16 + nib) * 8 + 4 * hh));
                        qj[0] += v.x;
                        qj[1] += v.y;
                        qj[2] += v.z;
                        qj[3] += v.w;
                    } else {
                        const uint32_t s = (word >> rho) & 0x40404040u;
#pragma unroll
                        for (int q = 0; q < 16; ++q) {
                            const uint4 pv = *reinterpret_cast<const uint4*>(pw + (((t * KK + kk) * 16 + q) * 8 + 4 * hh));
                            const int wq = q < 15 ? (1 << q) : -(1 << 15);
                            iq[0] += wq * __popc(s & pv.x);
                            iq[1] += wq * __popc(s & pv.y);
                            iq[2] += wq * __popc(s & pv.z);
                            iq[3] += wq * __popc(s & pv.w);
                        }
                    }
                }
            }
            const float2 kn = __half22float2(*reinterpret_cast<const __half2*>(tile + C::Tr::CODE_BYTES + 8 * g + 4 * rho));
            float vn = __half2float(*reinterpret_cast<const __half*>(tile + C::Tr::CODE_BYTES + 64 + 4 * g + 2 * rho));
            const bool valid = tl * 16 + tau < seq;
            float L[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int h = 4 * hh + k;
                const float y = MODE == 1 ? qj[k] : uq[h] * (float)(2 * iq[k] - tq[h]);
                L[k] = valid ? kn.x * (1.0f / 128.0f) * fmaf(kn.y, y, cb[k]) : -CUDART_INF_F;
            }
            if (!valid) vn = 0.f;

            // ---- online softmax (lazy reference, as in the tensor-core kernel)
            const bool above = (L[0] > m[0]) || (L[1] > m[1]) || (L[2] > m[2]) || (L[3] > m[3]);
            if (__any_sync(kFull, above)) {
                float al[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    float mx = L[k];
#pragma unroll
                    for (int sh = 2; sh <= 16; sh <<= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, sh));
                    const float mn = fmaxf(m[k], mx + kRescaleSlack);
                    al[k] = fast_exp2(m[k] - mn);
                    l[k] *= al[k];
                    m[k] = mn;
                }
                float ao[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) ao[k] = __shfl_xor_sync(kFull, al[k], 1);
#pragma unroll
                for (int h = 0; h < 8; ++h) {
                    const float f = (h >> 2) == hh ? al[h & 3] : ao[h & 3];   // static register index
#pragma unroll
                    for (int mm = 0; mm < 4; ++mm) acc[mm][h] *= f;
                }
            }
            float pv4[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float pk = fast_exp2(L[k] - m[k]);
                l[k] += pk;
                pv4[k] = pk * vn;
            }
            *reinterpret_cast<float4*>(wvw + tau * 8 + 4 * hh) = make_float4(pv4[0], pv4[1], pv4[2], pv4[3]);
            __syncwarp();

            // ---- P V: this lane's coordinates lane + 32 mm, all 8 heads
#pragma unroll
            for (int mm = 0; mm < 4; ++mm) {
                const int i = lane + 32 * mm, kk = i >> 4, gi = i & 7, r1 = (i >> 3) & 1;
                float cv[16];   // level of token 2t + 8 r2 + e
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const uint32_t word = *cc_word(tile, 4 * gi + t, 8 + kk);
#pragma unroll
                    for (int r2 = 0; r2 < 2; ++r2)
#pragma unroll
                        for (int e = 0; e < 2; ++e)
                            cv[2 * t + 8 * r2 + e] = vtab[(word >> (8 * (r1 + 2 * r2) + 4 * e)) & 15];
                }
#pragma unroll
                for (int tok = 0; tok < 16; ++tok) {
                    const float4 pa = *reinterpret_cast<const float4*>(wvw + tok * 8);
                    const float4 pb = *reinterpret_cast<const float4*>(wvw + tok * 8 + 4);
                    acc[mm][0] = fmaf(pa.x, cv[tok], acc[mm][0]);
                    acc[mm][1] = fmaf(pa.y, cv[tok], acc[mm][1]);
                    acc[mm][2] = fmaf(pa.z, cv[tok], acc[mm][2]);
                    acc[mm][3] = fmaf(pa.w, cv[tok], acc[mm][3]);
                    acc[mm][4] = fmaf(pb.x, cv[tok], acc[mm][4]);
                    acc[mm][5] = fmaf(pb.y, cv[tok], acc[mm][5]);
                    acc[mm][6] = fmaf(pb.z, cv[tok], acc[mm][6]);
                    acc[mm][7] = fmaf(pb.w, cv[tok], acc[mm][7]);
                }
            }
            __syncwarp();   // the tile's p |v| are read before the next tile writes them
        }

        // ---- merge the warps' states into the partial of slot c + u
#pragma unroll
        for (int k = 0; k < 4; ++k)
#pragma unroll
            for (int sh = 2; sh <= 16; sh <<= 1) l[k] += __shfl_xor_sync(kFull, l[k], sh);
        fence_proxy_async();
        __syncthreads();   // every warp is done with its ring: the merge buffer aliases it
        float* mw = mrg + (size_t)w * 8 * RS;
        const bool idle = w >= ntile;
        if (tau == 0) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                mw[(4 * hh + k) * RS] = idle ? -CUDART_INF_F : m[k];
                mw[(4 * hh + k) * RS + 1] = l[k];
            }
        }
#pragma unroll
        for (int mm = 0; mm < 4; ++mm)
#pragma unroll
            for (int h = 0; h < 8; ++h) mw[h * RS + 2 + lane + 32 * mm] = acc[mm][h];
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
        __syncthreads();   // tables, ring and merge buffer free for the next segment
        x = U0 + se;
    }
    while (consumed < issued) {
        if (!mbar_wait(bar_s + 8 * (consumed & 1u), (consumed >> 1) & 1u)) break;
        ++consumed;
    }
}
