// Coordinate pairing of the rotation.
//
// The block-diagonal rotation of Periodic RoPE §3.1 Eq. 2 turns coordinate
// pairs (2i, 2i+1) by p * theta_i (adjacent pairing). Many model
// implementations pair coordinate i with i + D/2 instead (half-split
// pairing). The two are the same rotation seen through a fixed permutation
// of the head dimensions: with pi(x) = (x_0, x_{D/2}, x_1, x_{D/2+1}, ...),
//   R_half(p) x = pi^-1 R_adjacent(p) pi x,
// and a score <R_a q, R_b k> is unchanged when both sides are permuted. So
// every attention kernel works in adjacent order; a half-split call permutes
// the query once on entry and its keys where they are rotated anyway (the key
// pre-pass, the cache writer). Caches of half-split keys are therefore kept
// in adjacent order (element 2i holds coordinate i, 2i+1 holds i + D/2);
// values and outputs keep their own order.
#pragma once

#include "common.cuh"

namespace ropeattn {

// Rotation pair i of a row of D bf16 values: (x_{2i}, x_{2i+1}) for adjacent
// pairing, (x_i, x_{i+D/2}) for half-split; row_word indexes the row's first
// 4-byte word and P = D/2.
__device__ __forceinline__ void load_rot_pair(const uint32_t* words, size_t row_word, int i, int P, bool half,
                                              float& x0, float& x1) {
  if (!half) {
    const uint32_t w = __ldg(words + row_word + i);
    x0 = bf16lo(w);
    x1 = bf16hi(w);
  } else {
    const unsigned short* h = reinterpret_cast<const unsigned short*>(words + row_word);
    x0 = __uint_as_float(static_cast<uint32_t>(__ldg(h + i)) << 16);
    x1 = __uint_as_float(static_cast<uint32_t>(__ldg(h + i + P)) << 16);
  }
}

// Rotation pairs 4c .. 4c+3 of a row, as rotate-ready values: x0[j], x1[j]
// are the pair 4c+j ((x_{2i}, x_{2i+1}) adjacent, (x_i, x_{i+D/2})
// half-split). One 16-byte load (adjacent) or two 8-byte loads (half-split);
// row_word indexes the row's first 4-byte word (16-byte aligned rows), P = D/2.
__device__ __forceinline__ void load_rot_quad(const uint32_t* words, size_t row_word, int c, int P, bool half,
                                              float (&x0)[4], float (&x1)[4]) {
  if (!half) {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(words + row_word) + c);
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      x0[j] = bf16lo(ww[j]);
      x1[j] = bf16hi(ww[j]);
    }
  } else {
    const uint2* g = reinterpret_cast<const uint2*>(words + row_word);
    const uint2 lo = __ldg(g + c);            // x_{4c} .. x_{4c+3}
    const uint2 hi = __ldg(g + P / 4 + c);    // x_{P+4c} .. x_{P+4c+3}
    x0[0] = bf16lo(lo.x); x0[1] = bf16hi(lo.x); x0[2] = bf16lo(lo.y); x0[3] = bf16hi(lo.y);
    x1[0] = bf16lo(hi.x); x1[1] = bf16hi(hi.x); x1[2] = bf16lo(hi.y); x1[3] = bf16hi(hi.y);
  }
}

// out[r] = pi(in[r]) for rows of D bf16 values: out[2i] = in[i],
// out[2i+1] = in[i + D/2]. Four pairs per thread: two 8-byte loads, one
// 16-byte store. Both buffers 16-byte aligned; D a multiple of 8.
struct PairInterleaveArgs {
  const uint2* in;   // rows x D bf16, as 8-byte groups of four values
  uint4* out;        // rows x D bf16, as 16-byte groups of eight values
  long long rows;
  int D;
};

__global__ void __launch_bounds__(256) pair_interleave_kernel(const PairInterleaveArgs a) {
  const int quads = a.D >> 3;   // groups of four pairs per row
  const long long g = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (g >= a.rows * quads) return;
  const long long r = g / quads;
  const int j = static_cast<int>(g % quads);
  const size_t base = static_cast<size_t>(r) * (a.D >> 2);   // row start in 8-byte groups
  const uint2 lo = __ldg(a.in + base + j);                    // x_{4j} .. x_{4j+3}
  const uint2 hi = __ldg(a.in + base + quads + j);            // x_{D/2+4j} .. x_{D/2+4j+3}
  uint4 o;
  o.x = (lo.x & 0xFFFFu) | (hi.x << 16);
  o.y = (lo.x >> 16) | (hi.x & 0xFFFF0000u);
  o.z = (lo.y & 0xFFFFu) | (hi.y << 16);
  o.w = (lo.y >> 16) | (hi.y & 0xFFFF0000u);
  a.out[static_cast<size_t>(r) * (a.D >> 3) + j] = o;
}

}  // namespace ropeattn
