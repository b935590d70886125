// Decode-cache writer (Jet-Long §3.2 Eq. 4): each new key is stored rotated
// at its own position, and the cache is never rewritten afterwards, however
// the bifocal group size G changes as the sequence grows.
//
// One thread per (token, four rotation pairs), as in the prefill key
// pre-pass: the angle p * theta_i is taken in double precision (p the kind's
// primary position of the token's absolute index), sincos in double, rounded
// to fp32; each pair is rotated in fp32 and rounded to bf16 (nearest even)
// for every (batch, kv head) row of the token. The value quad is copied
// alongside. Consecutive threads touch consecutive 16-byte groups of a row.
// Half-split keys are read pair (i, i + D/2) and stored in adjacent order
// (pairing.cuh).
#pragma once

#include "common.cuh"
#include "pairing.cuh"
#include "posmap.cuh"

namespace ropeattn {

struct CacheArgs {
  const uint32_t* k;   // [B, count, Hkv, D] bf16 pairs
  const uint32_t* v;   // same layout, or null
  uint32_t* k_cache;   // [B, cache_len, Hkv, D]
  uint32_t* v_cache;   // same layout, or null
  long long start, count, cache_len;
  int B, Hkv, D;
  int half;            // 1: k pairs coordinates (i, i + D/2)
  PosMap m;
  double theta[kMaxPairs];
};

// One thread per (token, four rotation pairs); the host launches
// ceil(count / (256 / (D/8))) blocks of 256 threads.
__global__ void __launch_bounds__(256) cache_write_kernel(const CacheArgs a) {
  const int P = a.D >> 1;
  const int Q = P >> 2;                       // four-pair chunks per row
  const int rows = blockDim.x / Q;
  const long long i_tok = static_cast<long long>(blockIdx.x) * rows + threadIdx.x / Q;
  const int c = threadIdx.x % Q;
  if (i_tok >= a.count) return;
  const long long t = a.start + i_tok;
  float cs[4] = {1.f, 1.f, 1.f, 1.f}, sn[4] = {0.f, 0.f, 0.f, 0.f};
  if (a.m.kind != kNope) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      double sd, cd;
      sincos(static_cast<double>(pos_primary(a.m, static_cast<int>(t))) * a.theta[4 * c + j], &sd, &cd);
      cs[j] = static_cast<float>(cd);
      sn[j] = static_cast<float>(sd);
    }
  }
#pragma unroll 4
  for (int bh = 0; bh < a.B * a.Hkv; ++bh) {
    const int b = bh / a.Hkv, h = bh % a.Hkv;
    const size_t src_row = ((static_cast<size_t>(b) * a.count + i_tok) * a.Hkv + h) * P;
    const size_t dst_row = ((static_cast<size_t>(b) * a.cache_len + t) * a.Hkv + h) * P;
    if (a.m.kind == kNope) {
      reinterpret_cast<uint4*>(a.k_cache + dst_row)[c] = __ldg(reinterpret_cast<const uint4*>(a.k + src_row) + c);
    } else {
      float x0[4], x1[4];
      load_rot_quad(a.k, src_row, c, P, a.half != 0, x0, x1);
      uint32_t y[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float y0, y1;
        rot_pair(x0[j], x1[j], cs[j], sn[j], y0, y1);
        y[j] = pack_bf16x2(y0, y1);
      }
      reinterpret_cast<uint4*>(a.k_cache + dst_row)[c] = make_uint4(y[0], y[1], y[2], y[3]);
    }
    if (a.v != nullptr)
      reinterpret_cast<uint4*>(a.v_cache + dst_row)[c] = __ldg(reinterpret_cast<const uint4*>(a.v + src_row) + c);
  }
}

// Unfused decode (comparator): the correction rotation of Jet-Long Eq. 5-6
// done as a separate pass over the cache instead of in the attention kernel.
// For a query at t, a remote key s (t - s > w0) scores
//   q_remote . R(Delta s) k_cache[s] = q_local . R(Delta s - Delta q) k_cache[s]
// (R_a R_b = R_{a+b}), so writing every remote key turned by
// Delta s - Delta q, and every local key unchanged, into a copy lets a
// standard-RoPE decode (query at p(t) = t, keys read as stored) give the
// bifocal scores. One thread per (key, pair), angles in double, fp32
// rotation, bf16 result.
struct UnfusedRotArgs {
  const uint32_t* k_cache;  // [B, n, Hkv, D]
  uint32_t* k_out;          // [B, n, Hkv, D]
  int B, n, Hkv, D, k_local, dq;
  PosMap m;
  double theta[kMaxPairs];
};

// One thread per (key, four rotation pairs); the host launches
// ceil(n / (256 / (D/8))) blocks of 256 threads.
__global__ void __launch_bounds__(256) unfused_rotate_kernel(const UnfusedRotArgs a) {
  const int P = a.D >> 1;
  const int Q = P >> 2;                       // four-pair chunks per row
  const int rows = blockDim.x / Q;
  const int s = blockIdx.x * rows + threadIdx.x / Q;
  const int c = threadIdx.x % Q;
  if (s >= a.n) return;
  const bool remote = s < a.k_local;
  float cs[4] = {1.f, 1.f, 1.f, 1.f}, sn[4] = {0.f, 0.f, 0.f, 0.f};
  if (remote) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      double sd, cd;
      sincos(static_cast<double>(pos_remote(a.m, s) - s - a.dq) * a.theta[4 * c + j], &sd, &cd);
      cs[j] = static_cast<float>(cd);
      sn[j] = static_cast<float>(sd);
    }
  }
#pragma unroll 4
  for (int bh = 0; bh < a.B * a.Hkv; ++bh) {
    const int b = bh / a.Hkv, h = bh % a.Hkv;
    const size_t row = ((static_cast<size_t>(b) * a.n + s) * a.Hkv + h) * P;
    const uint4 x = __ldg(reinterpret_cast<const uint4*>(a.k_cache + row) + c);
    uint4 y = x;
    if (remote) {
      const uint32_t xw[4] = {x.x, x.y, x.z, x.w};
      uint32_t yw[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float y0, y1;
        rot_pair(bf16lo(xw[j]), bf16hi(xw[j]), cs[j], sn[j], y0, y1);
        yw[j] = pack_bf16x2(y0, y1);
      }
      y = make_uint4(yw[0], yw[1], yw[2], yw[3]);
    }
    reinterpret_cast<uint4*>(a.k_out + row)[c] = y;
  }
}

}  // namespace ropeattn
