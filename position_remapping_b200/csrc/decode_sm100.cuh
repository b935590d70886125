// Definitions shared by the split-KV decode (decode_tc_sm100.cuh): the launch
// parameters, exact angles from fixed-point turns, and packed fp32x2 helpers.
#pragma once

#include "common.cuh"
#include "posmap.cuh"

namespace ropeattn {

struct DecodeParams {
  const __nv_bfloat16* q;  // [B, Hq, D]
  float* out;              // [B, Hq, D]
  float* lse;              // [B, Hq]
  float* part_o;           // [B, Hq, nsplit, D]
  float2* part_ml;         // [B, Hq, nsplit] (m in log2 units, l)
  int* counters;           // [B, Hkv]
  int B, n, Hq, Hkv;
  int nsplit, keys_per_split;
  int k_begin;             // first attended key (Periodic RoPE window), else 0
  int k_local;             // keys >= k_local are local (exact-position) keys
  int bifocal;             // 1 when keys are read through the correction rotation
  PosMap m;
  float scale_log2;
  unsigned long long turns[kMaxPairs];  // theta_i / (2 pi) mod 1, in units of 2^-64
};

// (cos, sin) of u * theta for an integer position u, with theta given as its
// fraction of a turn in 64-bit fixed point: the product modulo 2^64 is the
// angle modulo one turn, exactly; its top 32 bits, as a signed value, are the
// angle in half-turns in [-1, 1) for sincospi.
__device__ __forceinline__ float2 turn_cs(int u, unsigned long long turn) {
  const unsigned long long ph = turn * static_cast<unsigned long long>(static_cast<long long>(u));
  const float x = static_cast<float>(static_cast<int>(ph >> 32)) * 4.656612873077392578125e-10f;  // 2^-31
  float s, c;
  sincospif(x, &s, &c);
  return make_float2(c, s);
}

// Packed fp32x2 helpers (Blackwell FFMA2 / FMUL2).
__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 neg2(float2 a) { return make_float2(-a.x, -a.y); }

}  // namespace ropeattn
