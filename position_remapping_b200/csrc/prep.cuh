// Key pre-rotation and query angle tables for prefill.
//
// Every key tile is read by all S/128 query tiles of every query head of its
// group, so the keys are rotated once, here, in one streaming pass (per
// position map the kind uses), instead of once per tile visit. The same pass
// writes the (cos, sin) table of each query position that the attention
// kernel applies to the query tile it stages in shared memory.
//
// Angles: theta_i = base^(-2i/D) / s (Periodic RoPE §3.1 Eq. 1; position
// interpolation, Jet-Long §2.2), phase = p * theta_i in double precision,
// sincos in double, rounded to fp32. The rotation of a pair (Eq. 2) is done in
// fp32 and the result rounded to bf16 (nearest even), the tensor-core operand
// type. Half-split keys are read pair (i, i + D/2) and written in adjacent
// order (pairing.cuh).
#pragma once

#include "common.cuh"
#include "pairing.cuh"
#include "posmap.cuh"

namespace ropeattn {

struct PrepArgs {
  const uint32_t* k;      // [B, S, Hkv, D] bf16, read as bf16 pairs
  uint32_t* k_rot0;       // map 0: primary / local positions
  uint32_t* k_rot1;       // map 1: remote positions (BIFOCAL), else null
  float2* tab0;           // [S][D/2] (cos, sin) at map-0 positions
  float2* tab1;           // [S][D/2] at map-1 positions, or null
  int B, S, Hkv, D;
  int half;               // 1: k pairs coordinates (i, i + D/2)
  PosMap m;
  double theta[kMaxPairs];
};

// One thread per (token, four rotation pairs): the angles of its pairs
// under each map once, then for every (batch, head) row one 16-byte load of
// the key quad, rotated under every map, one 16-byte store per map. The
// host launches ceil(S / (256 / (D/8))) blocks of 256 threads.
__global__ void __launch_bounds__(256) rope_prep_kernel(const PrepArgs a) {
  const int P = a.D >> 1;
  const int Q = P >> 2;                       // four-pair chunks per row
  const int rows = blockDim.x / Q;
  const int t = blockIdx.x * rows + threadIdx.x / Q;
  const int c = threadIdx.x % Q;
  if (t >= a.S) return;
  const int nmaps = a.k_rot1 ? 2 : 1;
  float cs[2][4], sn[2][4];
  for (int mi = 0; mi < nmaps; ++mi) {
    const int p = mi == 0 ? pos_primary(a.m, t) : pos_remote(a.m, t);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      double sd, cd;
      sincos(static_cast<double>(p) * a.theta[4 * c + j], &sd, &cd);
      cs[mi][j] = static_cast<float>(cd);
      sn[mi][j] = static_cast<float>(sd);
    }
    float4* tab = reinterpret_cast<float4*>((mi == 0 ? a.tab0 : a.tab1) + static_cast<size_t>(t) * P + 4 * c);
    tab[0] = make_float4(cs[mi][0], sn[mi][0], cs[mi][1], sn[mi][1]);
    tab[1] = make_float4(cs[mi][2], sn[mi][2], cs[mi][3], sn[mi][3]);
  }
#pragma unroll 4
  for (int bh = 0; bh < a.B * a.Hkv; ++bh) {
    const int b = bh / a.Hkv, h = bh % a.Hkv;
    const size_t row = ((static_cast<size_t>(b) * a.S + t) * a.Hkv + h) * P;
    float x0[4], x1[4];
    load_rot_quad(a.k, row, c, P, a.half != 0, x0, x1);
    for (int mi = 0; mi < nmaps; ++mi) {
      uint32_t y[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float y0, y1;
        rot_pair(x0[j], x1[j], cs[mi][j], sn[mi][j], y0, y1);
        y[j] = pack_bf16x2(y0, y1);
      }
      uint32_t* dst = mi == 0 ? a.k_rot0 : a.k_rot1;
      reinterpret_cast<uint4*>(dst + row)[c] = make_uint4(y[0], y[1], y[2], y[3]);
    }
  }
}

// Prefill of a chunk of query rows against a decode cache (Jet-Long §3.2
// Eq. 4: the cache holds every key rotated at its own position). The cache
// is the local key tensor as it stands; for BIFOCAL this pass writes the
// remote keys R(Delta s) k_cache[s], Delta s = f(s) - s (the correction of
// Eq. 5-6), for every cached row, and the query angle tables of the chunk's
// rows (absolute positions start + r). One thread per (token, pair).
struct ChunkPrepArgs {
  const uint32_t* k_cache;  // [B, L, Hkv, D] bf16 pairs
  uint32_t* k_rem;          // [B, L, Hkv, D] remote keys (BIFOCAL), else null
  float2* tab0;             // [count][D/2] (cos, sin) at primary positions, or null (NOPE)
  float2* tab1;             // [count][D/2] at remote positions (BIFOCAL), else null
  int B, L, Hkv, D, start;
  long long cache_rows;     // rows between batch entries of k_cache (>= L)
  PosMap m;
  double theta[kMaxPairs];
};

// One thread per (token, four rotation pairs); the host launches
// ceil(L / (256 / (D/8))) blocks of 256 threads.
__global__ void __launch_bounds__(256) chunk_prep_kernel(const ChunkPrepArgs a) {
  const int P = a.D >> 1;
  const int Q = P >> 2;                       // four-pair chunks per row
  const int rows = blockDim.x / Q;
  const int t = blockIdx.x * rows + threadIdx.x / Q;
  const int c = threadIdx.x % Q;
  if (t >= a.L) return;
  if (a.k_rem != nullptr) {
    float cs[4], sn[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      double sd, cd;
      sincos(static_cast<double>(pos_remote(a.m, t) - t) * a.theta[4 * c + j], &sd, &cd);
      cs[j] = static_cast<float>(cd);
      sn[j] = static_cast<float>(sd);
    }
#pragma unroll 4
    for (int bh = 0; bh < a.B * a.Hkv; ++bh) {
      const int b = bh / a.Hkv, h = bh % a.Hkv;
      const size_t w = ((static_cast<size_t>(b) * a.L + t) * a.Hkv + h) * P;
      const size_t r = ((static_cast<size_t>(b) * a.cache_rows + t) * a.Hkv + h) * P;
      const uint4 x = __ldg(reinterpret_cast<const uint4*>(a.k_cache + r) + c);
      const uint32_t xw[4] = {x.x, x.y, x.z, x.w};
      uint32_t y[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float y0, y1;
        rot_pair(bf16lo(xw[j]), bf16hi(xw[j]), cs[j], sn[j], y0, y1);
        y[j] = pack_bf16x2(y0, y1);
      }
      reinterpret_cast<uint4*>(a.k_rem + w)[c] = make_uint4(y[0], y[1], y[2], y[3]);
    }
  }
  if (t >= a.start && a.tab0 != nullptr) {
    const size_t r = static_cast<size_t>(t - a.start) * P + 4 * c;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      double sd, cd;
      sincos(static_cast<double>(pos_primary(a.m, t)) * a.theta[4 * c + j], &sd, &cd);
      a.tab0[r + j] = make_float2(static_cast<float>(cd), static_cast<float>(sd));
      if (a.tab1 != nullptr) {
        sincos(static_cast<double>(pos_remote(a.m, t)) * a.theta[4 * c + j], &sd, &cd);
        a.tab1[r + j] = make_float2(static_cast<float>(cd), static_cast<float>(sd));
      }
    }
  }
}

}  // namespace ropeattn
