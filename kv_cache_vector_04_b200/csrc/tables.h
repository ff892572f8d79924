// Host tables of one TurboQuant context (codebooks, rotation signs, QJL matrix).
#pragma once
#include <cstdint>
#include <vector>

namespace tq {

// Most codebook levels of a format: 7-bit key cells (the 8-bit TurboQuant keys
// of k8v4, (7, 4, 1)).
constexpr int kMaxCellBits = 7;
constexpr int kMaxLevels = 1 << kMaxCellBits;

struct HostTables {
    int d = 0, bits = 0, m = 0, kbits = 0, vbits = 0, qjl = 1;
    int codebook = 0;                          // 0: N(0, 1/d) model, 1: exact Beta marginal
    std::vector<float> centroids_k, bounds_k;  // 2^kbits levels, 2^kbits - 1 edges (fp32)
    std::vector<float> centroids_v, bounds_v;  // 2^vbits levels, 2^vbits - 1 edges (fp32)
    std::vector<int8_t> signs;                 // D: d entries of +-1
    std::vector<float> S;                      // m x d row-major, fp16-exact values
    float alpha_k = 1.f;                       // fp16 decode scale of the key levels
};

// Lloyd–Max codebook for N(0, 1/d) with 2^B levels, rounded once to fp32;
// bounds are the fp32 midpoints of neighbouring levels. False if the fp64
// iteration did not converge.
bool build_codebook(int B, int d, float* centroids, float* bounds);
// The same for the exact marginal of a rotated unit-vector coordinate,
// (1 + y)/2 ~ Beta((d-1)/2, (d-1)/2), instead of its N(0, 1/d) limit.
bool build_codebook_beta(int B, int d, float* centroids, float* bounds);
void build_rotation_signs(int d, uint64_t seed, int8_t* signs);
void build_qjl_matrix(int m, int d, uint64_t seed, float* S);
// Tables of the format (kbits, vbits, qjl); TurboQuant at b bits is (b-1, b, 1).
// codebook: 0 = Lloyd–Max for N(0, 1/d), 1 = for the exact Beta marginal.
bool build_host_tables(int d, int kbits, int vbits, int qjl, int codebook, uint64_t seed,
                       HostTables& t);
// Scale in [1, 2) that puts alpha * sqrt(d) * c_j closest to fp16 values for
// the n/2 positive levels c_j (the kernel's decode table precision).
float choose_decode_scale(const float* centroids, int n, int d);

}  // namespace tq
