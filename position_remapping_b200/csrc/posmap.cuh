// Position maps. One definition, inlined by the position-map kernel, the key
// pre-rotation, the query-tile rotation and the decode kernel, so the
// positions every kernel uses are the ones ropeattn_posmap reports.
#pragma once

#include <stdint.h>

namespace ropeattn {

enum Kind : int { kStandard = 0, kEndPrompt = 1, kPeriodic = 2, kNope = 3, kBifocal = 4 };

struct PosMap {
  int kind;
  int seg1_len;    // EndPrompt n1
  int term_start;  // EndPrompt first terminal position
  int window;      // Periodic RoPE W
  int w0;          // Jet-Long local window
  int G;           // Jet-Long group size for this L (1 otherwise)
};

// Position RoPE uses for token t (Periodic RoPE §3.2 Eq. 4; EndPrompt
// two-segment positions; Jet-Long: the exact position for the local window).
__host__ __device__ __forceinline__ int pos_primary(const PosMap& m, int t) {
  switch (m.kind) {
    case kEndPrompt: return t < m.seg1_len ? t : m.term_start + (t - m.seg1_len);
    case kPeriodic: return t % m.window;
    case kNope: return 0;
    default: return t;
  }
}

// Jet-Long §3.1 Eq. 3: f(x) = floor(x / G).
__host__ __device__ __forceinline__ int pos_remote(const PosMap& m, int t) { return t / m.G; }

// Jet-Long §3.1 Eq. 2: G = max(1, ceil(L / w_pretrained)).
__host__ __device__ __forceinline__ int group_size(long long L, long long w_pretrained) {
  long long g = (L + w_pretrained - 1) / w_pretrained;
  return g < 1 ? 1 : static_cast<int>(g);
}

__global__ void posmap_kernel(PosMap m, int L, int32_t* __restrict__ out_local,
                              int32_t* __restrict__ out_remote) {
  int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= L) return;
  out_local[t] = pos_primary(m, t);
  if (out_remote) out_remote[t] = m.kind == kBifocal ? pos_remote(m, t) : t;
}

}  // namespace ropeattn
