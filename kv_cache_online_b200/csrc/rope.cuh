// Rotate-half RoPE angles for the CUDA-core kernels (iS-KV reading notes, Algorithm 3 step 8:
// every key is rotated by its own position; pairs (j, j + hd/2), angle pos * theta^(-2j/hd)).
//
// pos * theta^(-2j/hd) reaches tens of thousands of radians, where one float32 ulp is ~4e-3 rad.
// The angle is therefore formed and reduced modulo 2 pi in float64 and only the reduced angle
// (|a| <= pi) goes to sincosf.
#pragma once

#include "common.cuh"

namespace iskv {

ISKV_DEV double rope_inv_freq(int j, int hd, double log_theta) {
  return exp(-2.0 * (double)j / (double)hd * log_theta);
}

ISKV_DEV void rope_sincos(int64_t pos, double inv_freq, float &c, float &s) {
  const double two_pi = 6.283185307179586476925286766559;
  const double inv_two_pi = 0.15915494309189533576888376337251;
  double a = (double)pos * inv_freq;
  a = fma(-two_pi, rint(a * inv_two_pi), a);
  sincosf((float)a, &s, &c);
}

}  // namespace iskv
