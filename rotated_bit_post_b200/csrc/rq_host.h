// Host-side preparation routines (rotation tables, codebook, PCA basis).
#pragma once
#include <cstdint>
#include <vector>

namespace rq {

void make_rotation(int K, uint64_t seed, int8_t* sign, int32_t* perm, int32_t* rot);
uint8_t e4m3_encode(double v);
uint16_t float_to_bf16_rne(float f);
bool lloyd_max(int K, int levels, std::vector<double>& cent, std::vector<double>& bnd);
bool pca_basis(const uint16_t* calib, int n, int K, int r, uint16_t* U, double* evals);
void make_zigzag(const float* mag, int K, int block, int32_t* perm, int32_t* rot2);

}  // namespace rq
