// dequant.cuh -- reconstruction of cached tokens from the packed layout:
//   K'_j = bf16( (c_aj + (mn_g + code_j sc_g)) + sum_q U_jq (c8_q cs) )
//   V'_j = bf16(  c_bj + (mn_g + code_j sc_g) )
// (QuantWM, "Flickering after quantization?" (SynthePulse), PSAC paragraph:
// the Key is compensated when the cache is reconstructed; U is the basis
// version in force when the token was appended, c the centroid of the table
// version in force then.)
#pragma once
#include "common.cuh"

namespace qwm {

struct PackedHead {
  const uint8_t* k_codes;   // [tcap][d/4]
  const uint16_t* k_params; // [tcap][ng][2]
  const void* k_idx;        // [tcap]
  const int8_t* k_coef;     // [tcap][r]
  const uint16_t* k_cscale; // [tcap]
  const uint8_t* v_codes;
  const uint16_t* v_params;
  const void* v_idx;
  const uint16_t* cent_k;   // [C][d] of table version 0; version v at + v * cstride
  const uint16_t* cent_v;   // [C][d]
  const uint16_t* centver;  // [tcap] table version of each token
  size_t cstride;           // elements between table versions (H * C * d)
};

__device__ __forceinline__ PackedHead packed_head(const CacheView& v, const Dims& D, int h) {
  PackedHead p;
  const size_t base = (size_t)h * D.tcap;
  p.k_codes = v.k_codes + base * (D.d / 4);
  p.k_params = v.k_params + base * D.ng * 2;
  p.k_idx = (const uint8_t*)v.k_idx + base * D.idx_bytes;
  p.k_coef = v.k_coef + base * D.r;
  p.k_cscale = v.k_cscale + base;
  p.v_codes = v.v_codes + base * (D.d / 4);
  p.v_params = v.v_params + base * D.ng * 2;
  p.v_idx = (const uint8_t*)v.v_idx + base * D.idx_bytes;
  p.cent_k = v.cent_k + (size_t)h * D.C * D.d;
  p.cent_v = v.cent_v + (size_t)h * D.C * D.d;
  p.centver = v.centver;
  p.cstride = cent_slot_elems(D);
  return p;
}

__device__ __forceinline__ int load_idx(const void* idx, int64_t t, int idx_bytes) {
  return idx_bytes == 1 ? (int)((const uint8_t*)idx)[t] : (int)((const uint16_t*)idx)[t];
}

__device__ __forceinline__ float deq_int2(const uint8_t* codes, const uint16_t* params, int64_t t,
                                          int j, int d, int ng, int G) {
  int code = (codes[t * (d / 4) + j / 4] >> (2 * (j % 4))) & 3;
  const uint16_t* pr = params + (t * ng + j / G) * 2;
  return fmaf((float)code, h2f(pr[1]), h2f(pr[0]));
}

// K' element (fp32 before the bf16 rounding); U_h = basis of this head for the
// token's version ([d][r]).
__device__ __forceinline__ float key_elem(const PackedHead& p, const Dims& D, const float* U_h,
                                          int64_t t, int j) {
  int a = load_idx(p.k_idx, t, D.idx_bytes);
  const uint16_t* ck = p.cent_k + (size_t)p.centver[t] * p.cstride;
  float v = bf2f(ck[(size_t)a * D.d + j]) + deq_int2(p.k_codes, p.k_params, t, j, D.d, D.ng, D.G);
  if (D.r > 0) {
    float cs = h2f(p.k_cscale[t]);
    float corr = 0.0f;
    const int8_t* cf = p.k_coef + t * D.r;
    for (int q = 0; q < D.r; ++q) corr = fmaf(U_h[(size_t)j * D.r + q], (float)cf[q] * cs, corr);
    v += corr;
  }
  return v;
}

__device__ __forceinline__ float value_elem(const PackedHead& p, const Dims& D, int64_t t, int j) {
  int b = load_idx(p.v_idx, t, D.idx_bytes);
  const uint16_t* cv = p.cent_v + (size_t)p.centver[t] * p.cstride;
  return bf2f(cv[(size_t)b * D.d + j]) + deq_int2(p.v_codes, p.v_params, t, j, D.d, D.ng, D.G);
}

__device__ __forceinline__ const float* basis_of(const CacheView& v, const Dims& D, int ver, int h) {
  return v.basis + ((size_t)ver * D.H + h) * D.d * (D.r > 0 ? D.r : 1);
}

}  // namespace qwm
