// Host-side float64 builders for the codec constants (internal to libtq).
#pragma once

#include <cstddef>
#include <cstdint>
#include <vector>

namespace tqhost {

// n standard normals from SplitMix64 (counter form) + Box-Muller, row-major.
void gaussian_fill(uint64_t seed, size_t n, double* out);

// Q factor (row-major n x n) of the Householder QR of A, signed so diag(R) > 0.
std::vector<double> orthogonal_factor(const std::vector<double>& A, int n);

struct LloydMax {
  std::vector<double> centroids;   // 2^bits, ascending, antisymmetric
  std::vector<double> boundaries;  // 2^bits - 1 midpoints
  double distortion;               // per-coordinate MSE
};

// Lloyd-Max quantizer of the Beta((d-1)/2,(d-1)/2) law on [-1, 1].
LloydMax lloyd_max(int d, int bits);

// Lloyd-Max quantizer of the level-`level` angle law of the recursive polar
// form (level 1 uniform on [-pi, pi]; level l > 1 on [0, pi/2] with
// sin^2 phi ~ Beta(k/2, k/2), k = 2^(l-1)); symmetric about the centre.
LloydMax polar_angle_lloyd_max(int level, int bits);

}  // namespace tqhost
