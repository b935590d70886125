// The literal inclusion-exclusion merge of the three-call bifocal prefill
// (Jet-Long §3.3 Eq. 7), as a separate kernel: the comparator of the fused
// two-pass kernel. Per query row, with l_X the natural-log LSE of call X:
//   M = max(l_A, l_B, l_C),  W_X = exp(l_X - M),
//   O = (W_A O_A + W_B O_B - W_C O_C) / (W_A + W_B - W_C),
//   l = M + ln(W_A + W_B - W_C),
// all in fp32. One warp per (batch, position, head) row; each lane merges the
// float4 groups lane, lane + 32, ... of the row (D / 4 groups: 16, 32 or 64).
// O_B and l_B live in the output buffers and are overwritten in place.
#pragma once

#include "common.cuh"

namespace ropeattn {

struct MergeArgs {
  const float* oA;   // [B, S, Hq, D]
  const float* oC;
  float* out;        // O_B in, O out
  const float* lA;   // [B, Hq, S]
  const float* lC;
  float* lse;        // l_B in, l out
  long long rows;    // B * S * Hq
  int S, Hq, D;
};

__global__ void __launch_bounds__(256) three_call_merge_kernel(const MergeArgs a) {
  const long long row = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= a.rows) return;
  const int h = static_cast<int>(row % a.Hq);
  const long long bt = row / a.Hq;
  const int t = static_cast<int>(bt % a.S);
  const long long b = bt / a.S;
  const size_t li = (static_cast<size_t>(b) * a.Hq + h) * a.S + t;
  const float la = a.lA[li], lb = a.lse[li], lc = a.lC[li];
  const float M = fmaxf(fmaxf(la, lb), lc);
  const float wa = expf(la - M), wb = expf(lb - M), wc = expf(lc - M);
  const float den = wa + wb - wc;
  const float inv = 1.0f / den;
  const size_t base = static_cast<size_t>(row) * a.D;
  for (int c = lane * 4; c < a.D; c += 128) {
    const float4 xa = *reinterpret_cast<const float4*>(a.oA + base + c);
    const float4 xb = *reinterpret_cast<const float4*>(a.out + base + c);
    const float4 xc = *reinterpret_cast<const float4*>(a.oC + base + c);
    float4 o;
    o.x = (wa * xa.x + wb * xb.x - wc * xc.x) * inv;
    o.y = (wa * xa.y + wb * xb.y - wc * xc.y) * inv;
    o.z = (wa * xa.z + wb * xb.z - wc * xc.z) * inv;
    o.w = (wa * xa.w + wb * xb.w - wc * xc.w) * inv;
    *reinterpret_cast<float4*>(a.out + base + c) = o;
  }
  __syncwarp();
  if (lane == 0) a.lse[li] = M + logf(den);
}

}  // namespace ropeattn
