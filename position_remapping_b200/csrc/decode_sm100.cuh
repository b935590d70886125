// One decode step over an untouched RoPE key cache (Jet-Long §3.2), sm_100a.
//
// Split-KV: CTA (split, kv head, batch) owns a contiguous key range of one KV
// head. Warp 8 streams that range through shared memory with TMA, 32 keys per
// stage (no swizzle, no multicast); warps 0-7 consume it, each lane group of
// 8 lanes taking one key per stage with two 16-byte shared loads per lane.
//
// Scores: the query is rotated once to its position p(n-1) in fp32. For the
// bifocal map, keys with (n-1) - k > w0 are read through the correction
// rotation of Eq. 6, k_remote = R(Delta k) k_cache[k] with
// Delta k = floor(k/G) - k = -u(k), against the query corrected by
// Delta q = floor((n-1)/G) - (n-1). Each lane carries the phasors
// exp(i u(k) theta_i) of its pairs and advances them from one key of its
// stream to the next (32 positions apart) by one complex multiply; they are
// re-seeded exactly (argument reduced in double) every 32 stages.
//
// Each lane group keeps an online softmax per query head of the GQA group;
// the CTA merges its groups and warps, writes (O, m, l) for its split, and the
// last CTA of the (batch, kv head) to arrive merges all splits in split order.
#pragma once

#include "common.cuh"
#include "posmap.cuh"

namespace ropeattn {

constexpr int kDecKeys = 32;         // keys per stage
constexpr int kDecStages = 6;        // ring depth
constexpr int kDecConsumerWarps = 8;
constexpr int kDecThreads = (kDecConsumerWarps + 1) * 32;
constexpr int kDecReseed = 32;       // stages between exact phasor re-seeds

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
  int k_local;             // keys >= k_local are read without correction
  int bifocal;             // 1 when remote keys need the correction rotation
  PosMap m;
  float scale_log2;
  double theta[kMaxPairs];
};

// (cos, sin) of phase * theta, with the argument reduced modulo 2*pi in double
// before the fp32 sincos.
__device__ __forceinline__ float2 phase_cs(double phase) {
  const double two_pi = 6.283185307179586476925286766559;
  const double r = phase - two_pi * rint(phase * (1.0 / two_pi));
  float s, c;
  sincosf(static_cast<float>(r), &s, &c);
  return make_float2(c, s);
}

template <int D>
struct DecodeSmem {
  static constexpr int kRowBytes = D * 2;
  static constexpr int kStageBytes = 2 * kDecKeys * kRowBytes;  // K then V
  static constexpr int kRing = kDecStages * kStageBytes;
  static constexpr int kBar = kRing;                             // full[], empty[]
  static constexpr int kMisc = kBar + 2 * kDecStages * 8;       // abort flag, last flag
  static constexpr int kTotal = kMisc + 16;
};

template <int D, int GRP>
__global__ void __launch_bounds__(kDecThreads)
    decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const DecodeParams p) {
  using L = DecodeSmem<D>;
  constexpr int NV = D / 64;         // 16-byte vectors per lane per row
  constexpr int NE = 8 * NV;         // elements per lane
  constexpr int NP = 4 * NV;         // rotation pairs per lane

  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* empty = full + kDecStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc);
  volatile int* last_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int split = blockIdx.x;
  const int hkv = blockIdx.y;
  const int b = blockIdx.z;

  const int kb = min(p.n, p.k_begin + split * p.keys_per_split);
  const int ke = min(p.n, kb + p.keys_per_split);
  const int nstage = (ke - kb + kDecKeys - 1) / kDecKeys;

  if (tid == 0) {
    for (int i = 0; i < kDecStages; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, kDecConsumerWarps);
    }
    *abort_flag = 0;
    *last_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();

  if (warp == kDecConsumerWarps) {
    // ---------------------------------------------------------------- TMA
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      for (int st = 0; st < nstage; ++st) {
        const int slot = st % kDecStages;
        if (!mbar_wait(empty + slot, ((st / kDecStages) & 1) ^ 1, abort_flag)) break;
        uint8_t* dst = smem + slot * L::kStageBytes;
        mbar_arrive_expect_tx(full + slot, L::kStageBytes);
        tma_load_4d(dst, &tmK, full + slot, 0, hkv, kb + st * kDecKeys, b);
        tma_load_4d(dst + kDecKeys * L::kRowBytes, &tmV, full + slot, 0, hkv, kb + st * kDecKeys, b);
      }
    }
  } else {
    // ----------------------------------------------------------- consumers
    const int j4 = lane >> 3;             // lane group within the warp
    const int l8 = lane & 7;              // lane within the group
    const int ks = warp * 4 + j4;         // key stream 0..31 == row in a stage
    const int t = p.n - 1;                // query position index
    // element e of this lane is dimension 64*(e/8) + 8*l8 + e%8; pair e/2
    auto pair_index = [&](int pp) { return 32 * (pp >> 2) + 4 * l8 + (pp & 3); };

    // query: rotate to p(t) (the local view) and, for the bifocal map, apply
    // the correction Delta q on top (the remote view, Eq. 5-6). Only one view
    // is held in registers; a stream switches from remote to local once.
    float qc[GRP][NE];
    auto load_query = [&](bool remote_view) {
      const int pq = pos_primary(p.m, t);
      const int dq = pos_remote(p.m, t) - t;
#pragma unroll
      for (int gi = 0; gi < GRP; ++gi) {
        const int hq = hkv * GRP + gi;
        const uint4* qs = reinterpret_cast<const uint4*>(p.q + (static_cast<size_t>(b) * p.Hq + hq) * D);
#pragma unroll
        for (int v = 0; v < NV; ++v) {
          const uint4 xq = __ldg(qs + v * 8 + l8);
          const uint32_t xw[4] = {xq.x, xq.y, xq.z, xq.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int pp = v * 4 + e;
            const double th = p.theta[pair_index(pp)];
            float a0 = bf16lo(xw[e]), a1 = bf16hi(xw[e]);
            if (p.m.kind != kNope) {
              const float2 cs = phase_cs(static_cast<double>(pq) * th);
              rot_pair(bf16lo(xw[e]), bf16hi(xw[e]), cs.x, cs.y, a0, a1);
            }
            if (remote_view) {
              const float2 cd = phase_cs(static_cast<double>(dq) * th);
              const float b0 = a0, b1 = a1;
              rot_pair(b0, b1, cd.x, cd.y, a0, a1);
            }
            qc[gi][2 * pp] = a0;
            qc[gi][2 * pp + 1] = a1;
          }
        }
      }
    };
    bool q_remote = p.bifocal && (kb + ks) < p.k_local;
    load_query(q_remote);

    // phasors exp(i u theta) for this lane's pairs, u(k) = k - floor(k/G)
    const int G = p.m.G;
    const int step_lo = kDecKeys - kDecKeys / G;  // u(k+32) - u(k) is step_lo or step_lo - 1
    float2 ph[NP], mul_a[NP], mul_b[NP];
    auto useed = [&](int k) { return k - k / G; };
    auto reseed = [&](int k) {
      const int u = useed(k);
#pragma unroll
      for (int pp = 0; pp < NP; ++pp) ph[pp] = phase_cs(static_cast<double>(u) * p.theta[pair_index(pp)]);
    };
    if (p.bifocal) {
#pragma unroll
      for (int pp = 0; pp < NP; ++pp) {
        const double th = p.theta[pair_index(pp)];
        mul_a[pp] = phase_cs(static_cast<double>(step_lo) * th);
        mul_b[pp] = phase_cs(static_cast<double>(step_lo - 1) * th);
      }
      reseed(kb + ks);
    }

    float m_run[GRP], l_run[GRP], acc[GRP][NE];
#pragma unroll
    for (int gi = 0; gi < GRP; ++gi) {
      m_run[gi] = -INFINITY;
      l_run[gi] = 0.f;
#pragma unroll
      for (int e = 0; e < NE; ++e) acc[gi][e] = 0.f;
    }

    bool ok = true;
    for (int st = 0; st < nstage; ++st) {
      const int slot = st % kDecStages;
      ok = __all_sync(0xffffffffu, mbar_wait(full + slot, (st / kDecStages) & 1, abort_flag));
      if (!ok) break;
      const uint8_t* row = smem + slot * L::kStageBytes + ks * L::kRowBytes;
      uint4 kv[NV], vv[NV];
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        kv[v] = *reinterpret_cast<const uint4*>(row + v * 128 + l8 * 16);
        vv[v] = *reinterpret_cast<const uint4*>(row + kDecKeys * L::kRowBytes + v * 128 + l8 * 16);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty + slot);

      const int k = kb + st * kDecKeys + ks;
      const bool valid = k < ke;                      // rows past the range are ignored
      const bool remote = p.bifocal && k < p.k_local;
      if (q_remote && !remote) {                      // this stream reached the local window
        load_query(false);
        q_remote = false;
      }
      float x[NE];
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        const uint32_t w[4] = {kv[v].x, kv[v].y, kv[v].z, kv[v].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          x[v * 8 + 2 * e] = bf16lo(w[e]);
          x[v * 8 + 2 * e + 1] = bf16hi(w[e]);
        }
      }
      if (remote) {
        // k_remote = R(-u theta) k_cache: (x0 c + x1 s, -x0 s + x1 c)
#pragma unroll
        for (int pp = 0; pp < NP; ++pp) {
          const float x0 = x[2 * pp], x1 = x[2 * pp + 1];
          x[2 * pp] = fmaf(x0, ph[pp].x, x1 * ph[pp].y);
          x[2 * pp + 1] = fmaf(x1, ph[pp].x, -x0 * ph[pp].y);
        }
      }
      float sc[GRP];
#pragma unroll
      for (int gi = 0; gi < GRP; ++gi) {
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < NE; ++e) a = fmaf(qc[gi][e], x[e], a);
        a += __shfl_xor_sync(0xffffffffu, a, 1);
        a += __shfl_xor_sync(0xffffffffu, a, 2);
        a += __shfl_xor_sync(0xffffffffu, a, 4);
        sc[gi] = a * p.scale_log2;
      }
      if (valid) {
        float vf[NE];
#pragma unroll
        for (int v = 0; v < NV; ++v) {
          const uint32_t w[4] = {vv[v].x, vv[v].y, vv[v].z, vv[v].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            vf[v * 8 + 2 * e] = bf16lo(w[e]);
            vf[v * 8 + 2 * e + 1] = bf16hi(w[e]);
          }
        }
#pragma unroll
        for (int gi = 0; gi < GRP; ++gi) {
          if (sc[gi] > m_run[gi]) {
            const float corr = ex2(m_run[gi] - sc[gi]);
            l_run[gi] *= corr;
#pragma unroll
            for (int e = 0; e < NE; ++e) acc[gi][e] *= corr;
            m_run[gi] = sc[gi];
          }
          const float pr = ex2(sc[gi] - m_run[gi]);
          l_run[gi] += pr;
#pragma unroll
          for (int e = 0; e < NE; ++e) acc[gi][e] = fmaf(pr, vf[e], acc[gi][e]);
        }
        // advance this stream's phasors to its next key (32 positions on)
        const int kn = k + kDecKeys;
        if (p.bifocal && kn < p.k_local && kn < ke) {
          if (((st + 1) % kDecReseed) == 0) {
            reseed(kn);
          } else {
            const bool a_step = (useed(kn) - useed(k)) == step_lo;
#pragma unroll
            for (int pp = 0; pp < NP; ++pp) {
              const float2 mm = a_step ? mul_a[pp] : mul_b[pp];
              const float c = ph[pp].x * mm.x - ph[pp].y * mm.y;
              const float s = ph[pp].x * mm.y + ph[pp].y * mm.x;
              ph[pp] = make_float2(c, s);
            }
          }
        }
      }
    }

    // ------------------------------------------- merge lane groups of a warp
#pragma unroll
    for (int gi = 0; gi < GRP; ++gi) {
#pragma unroll
      for (int off = 8; off <= 16; off <<= 1) {
        const float mo = __shfl_xor_sync(0xffffffffu, m_run[gi], off);
        const float lo = __shfl_xor_sync(0xffffffffu, l_run[gi], off);
        const float M = fmaxf(m_run[gi], mo);
        const float a = (l_run[gi] > 0.f) ? ex2(m_run[gi] - M) : 0.f;
        const float c = (lo > 0.f) ? ex2(mo - M) : 0.f;
#pragma unroll
        for (int e = 0; e < NE; ++e) {
          const float ao = __shfl_xor_sync(0xffffffffu, acc[gi][e], off);
          acc[gi][e] = acc[gi][e] * a + ao * c;
        }
        l_run[gi] = l_run[gi] * a + lo * c;
        m_run[gi] = M;
      }
    }
    // ------------------------------------------------ merge warps via smem
    // (the stage ring is free: every stage issued was consumed above)
    named_barrier_sync(1, kDecConsumerWarps * 32);
    float* red_o = reinterpret_cast<float*>(smem);                       // [8][GRP][D]
    float2* red_ml = reinterpret_cast<float2*>(smem + kDecConsumerWarps * GRP * D * 4);  // [8][GRP]
    if (j4 == 0) {
#pragma unroll
      for (int gi = 0; gi < GRP; ++gi) {
#pragma unroll
        for (int e = 0; e < NE; ++e) red_o[(warp * GRP + gi) * D + 64 * (e >> 3) + 8 * l8 + (e & 7)] = acc[gi][e];
        if (l8 == 0) red_ml[warp * GRP + gi] = make_float2(m_run[gi], l_run[gi]);
      }
    }
    named_barrier_sync(1, kDecConsumerWarps * 32);
    for (int idx = tid; idx < GRP * D; idx += kDecConsumerWarps * 32) {
      const int gi = idx / D, d = idx % D;
      float M = -INFINITY;
      for (int w = 0; w < kDecConsumerWarps; ++w) {
        const float2 ml = red_ml[w * GRP + gi];
        if (ml.y > 0.f) M = fmaxf(M, ml.x);
      }
      float o = 0.f, l = 0.f;
      for (int w = 0; w < kDecConsumerWarps; ++w) {
        const float2 ml = red_ml[w * GRP + gi];
        if (ml.y > 0.f) {
          const float f = ex2(ml.x - M);
          o = fmaf(red_o[(w * GRP + gi) * D + d], f, o);
          l = fmaf(ml.y, f, l);
        }
      }
      const int hq = hkv * GRP + gi;
      const size_t slot = (static_cast<size_t>(b) * p.Hq + hq) * p.nsplit + split;
      p.part_o[slot * D + d] = o;
      if (d == 0) p.part_ml[slot] = make_float2(M, l);
    }
    __threadfence();
    named_barrier_sync(1, kDecConsumerWarps * 32);
    if (tid == 0) {
      const int prev = atomicAdd(p.counters + b * p.Hkv + hkv, 1);
      *last_flag = (prev == p.nsplit - 1) ? 1 : 0;
    }
    named_barrier_sync(1, kDecConsumerWarps * 32);
    if (*last_flag) {
      // last CTA of this (batch, kv head): merge every split, in split order
      __threadfence();
      for (int idx = tid; idx < GRP * D; idx += kDecConsumerWarps * 32) {
        const int gi = idx / D, d = idx % D;
        const int hq = hkv * GRP + gi;
        const size_t base = (static_cast<size_t>(b) * p.Hq + hq) * p.nsplit;
        float M = -INFINITY;
        for (int s = 0; s < p.nsplit; ++s) {
          const float2 ml = __ldcg(p.part_ml + base + s);
          if (ml.y > 0.f) M = fmaxf(M, ml.x);
        }
        float o = 0.f, l = 0.f;
        for (int s = 0; s < p.nsplit; ++s) {
          const float2 ml = __ldcg(p.part_ml + base + s);
          if (ml.y > 0.f) {
            const float f = ex2(ml.x - M);
            o = fmaf(__ldcg(p.part_o + (base + s) * D + d), f, o);
            l = fmaf(ml.y, f, l);
          }
        }
        p.out[(static_cast<size_t>(b) * p.Hq + hq) * D + d] = o / l;
        if (d == 0) p.lse[static_cast<size_t>(b) * p.Hq + hq] = (M + __log2f(l)) * 0.69314718055994530942f;
      }
      if (tid == 0) p.counters[b * p.Hkv + hkv] = 0;
    }
    (void)ok;
  }
  __syncthreads();
  if (*abort_flag) {
    const unsigned long long t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 20000000ull) __nanosleep(100000);
  }
}

}  // namespace ropeattn
