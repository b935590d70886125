// Backward of the prefill (gradients of q, k, v through the routed softmax
// and both rotation maps), sm_100a, head_dim 64 and 128.
//
// With P the row softmax of scale * score(t,s) over the allowed keys,
// score(t,s) = <R_a q_t, R_b k_s> ((a, b) the positions the kind assigns; for
// the bifocal map (t, s) inside the local window and (f(t), f(s)) outside it,
// Jet-Long §3 Eq. 1), dO the upstream gradient of the output and
// Delta_t = dO_t . O_t:
//   dP(t,s) = dO_t . v_s,   dS(t,s) = P(t,s) (dP(t,s) - Delta_t),
//   dv_s = sum_t P(t,s) dO_t,
//   dk_s = scale * R_b^T sum_t dS(t,s) R_a q_t,
//   dq_t = scale * R_a^T sum_s dS(t,s) R_b k_s,
// the sums split by map for the bifocal kind. P is recomputed from the saved
// log-sum-exp of the forward: P = exp(scale * score - lse).
//
// Two kernels, neither with atomics, so results are bitwise reproducible:
//   bwd_dkdv_kernel  one CTA per 128-key tile of one (batch, kv head): loops
//                    over the query heads of the group and the 64-row query
//                    tiles that attend the tile, per map;
//                    S^T = K_r Q_r^T and dP^T = V dO^T on tcgen05 (keys as M),
//                    P^T and dS^T in fp32 by the softmax warps (lane = key),
//                    written back to TMEM as bf16, then dV += P^T dO and
//                    dK += dS^T Q_r with A read from TMEM.
//   bwd_dq_kernel    one CTA per 128-row query tile of one (batch, query head):
//                    loops over 64-key tiles per map; S = Q_r K_r^T,
//                    dP = dO V^T, dS (lane = query) back to TMEM as bf16,
//                    dQ += dS K_r.
// Rotated queries and keys (R_a q, R_b k, rounded to bf16 as the forward's
// operands) and the (cos, sin) tables per map come from the forward's
// streaming pre-rotation; the gradients of the rotated operands are turned
// back by R^T in fp32 in the epilogue. A bifocal CTA runs the remote map's
// pass first, parks its gradient (turned back) in the output rows, and adds
// it in the local pass's epilogue, as the forward parks its remote partial.
//
// Warps of both kernels: 0-3 and 4-7 the two softmax warpgroups (each owns
// half of the 64 columns of a score tile and half of the accumulator columns
// in the epilogue; TMEM lane = row), 8 TMA producer, 9 and 10 issue the two
// score-side MMAs (S and dP), 11 issues the gradient MMAs. TMEM (512
// columns): kernel A S[2] at [0,64) and [64,128), dP[2] at [128,256), then
// dV and dK, D columns each (three sets at D = 64, where they fit); kernel B
// three sets, S[3] at [0,192), dP[3] at [192,384), then dQ (a third set fits
// beside one accumulator). The bf16
// P and dS of a warpgroup's 32 columns are packed into the first 16 of those
// columns, where only that warpgroup reads the fp32 scores.
#pragma once

#include "common.cuh"
#include "pairing.cuh"
#include "posmap.cuh"
#include "prefill_sm100.cuh"

namespace ropeattn {

constexpr int kBwdThreads = 384;
constexpr int kBwdN = 64;       // the 64-wide side of every score tile
constexpr int kBwdWarpTMA = 8, kBwdWarpS = 9, kBwdWarpDP = 10, kBwdWarpG = 11;

// TMEM column of the bf16 operand (P or dS) for K step kk (16 columns of the
// score tile): warpgroup 0 packs columns 0-31 into [0,16), warpgroup 1
// columns 32-63 into [32,48)
__device__ __forceinline__ uint32_t bwd_pcol(int kk) { return (kk >> 1) * 32 + (kk & 1) * 8; }

struct BwdParams {
  float* dq;             // [B, S, Hq, D]
  float* dk;             // [B, S, Hkv, D]
  float* dv;             // [B, S, Hkv, D]
  const float* nlse2;    // [B, Hq, Sp] minus the forward log-sum-exp times log2(e)
  const float* ndelta;   // [B, Hq, Sp] minus rowsum(dO * O)
  const float2* tab0;    // [S][D/2] (cos, sin) at map-0 positions (null for NoPE)
  const float2* tab1;    // [S][D/2] at remote positions (bifocal)
  int B, S, Hq, Hkv;
  int Sp;                // row stride of nlse2 and ndelta: S rounded up to 64 (aligned bulk copies)
  int nkt, nqt;          // 128-row key tiles / query tiles per sequence
  int kind, window, w0;
  float scale_log2;      // softmax scale * log2(e)
  float scale;
  int half;              // half-split pairing: dq and dk in the heads' own order
};

// Allowed bands of the kind (distance t - s in [hi, lo]) with the map each
// band uses (0: main or local positions, 1: remote positions); bifocal: the
// remote band first, then the local one.
__device__ __forceinline__ int bwd_bands(const BwdParams& p, int (*bands)[3]) {
  if (p.kind == kBifocal) {
    bands[0][0] = kInf; bands[0][1] = p.w0 + 1; bands[0][2] = 1;
    bands[1][0] = p.w0; bands[1][1] = 0; bands[1][2] = 0;
    return 2;
  }
  bands[0][0] = p.kind == kPeriodic ? p.window - 1 : kInf;
  bands[0][1] = 0;
  bands[0][2] = 0;
  return 1;
}

// R^T (the rotation by minus the angle) of one pair, from the table entry
// (cos, sin) of the forward's angle.
__device__ __forceinline__ void unrot_pair(float y0, float y1, float c, float s, float& x0, float& x1) {
  x0 = __fmaf_rn(y0, c, __fmul_rn(y1, s));
  x1 = __fmaf_rn(y1, c, -__fmul_rn(y0, s));
}

// Writes half a gradient row: the D/2 fp32 values g of adjacent-order
// columns [c0, c0 + D/2) (already turned back and scaled) into the row `dst`,
// adding the parked value when `add`; for half-split pairing element pairs
// (2i, 2i+1) go to coordinates (i, i + D/2).
template <int D>
__device__ __forceinline__ void store_grad_half(float* dst, const float* g, int c0, bool add, bool half) {
  if (!half) {
#pragma unroll
    for (int e = 0; e < D / 2; e += 4) {
      float4 o = make_float4(g[e], g[e + 1], g[e + 2], g[e + 3]);
      if (add) {
        const float4 pr = *reinterpret_cast<const float4*>(dst + c0 + e);
        o.x += pr.x; o.y += pr.y; o.z += pr.z; o.w += pr.w;
      }
      *reinterpret_cast<float4*>(dst + c0 + e) = o;
    }
  } else {
    const int i0 = c0 / 2;
#pragma unroll
    for (int i = 0; i < D / 4; i += 4) {
      float4 lo = make_float4(g[2 * i], g[2 * i + 2], g[2 * i + 4], g[2 * i + 6]);
      float4 hi = make_float4(g[2 * i + 1], g[2 * i + 3], g[2 * i + 5], g[2 * i + 7]);
      if (add) {
        const float4 a = *reinterpret_cast<const float4*>(dst + i0 + i);
        const float4 c = *reinterpret_cast<const float4*>(dst + D / 2 + i0 + i);
        lo.x += a.x; lo.y += a.y; lo.z += a.z; lo.w += a.w;
        hi.x += c.x; hi.y += c.y; hi.z += c.z; hi.w += c.w;
      }
      *reinterpret_cast<float4*>(dst + i0 + i) = lo;
      *reinterpret_cast<float4*>(dst + D / 2 + i0 + i) = hi;
    }
  }
}

// Reads D/2 accumulator columns [c0, c0 + D/2) of this thread's TMEM lane,
// scales them, and for a rotating kind turns each pair back by the table
// entry of position row `pos` (R^T of the forward's rotation).
template <int D>
__device__ __forceinline__ void grad_half_from_tmem(uint32_t taddr, float scale, const float2* tab, int c0,
                                                    float (&g)[D / 2]) {
  uint32_t rr[32];
#pragma unroll
  for (int c = 0; c < D / 64; ++c) {
    tmem_ld32(taddr + c0 + c * 32, rr);
    tmem_ld_wait();
#pragma unroll
    for (int e = 0; e < 32; ++e) g[c * 32 + e] = __uint_as_float(rr[e]) * scale;
  }
  if (tab != nullptr) {
#pragma unroll
    for (int i = 0; i < D / 4; ++i) {
      const float2 cs = __ldg(tab + c0 / 2 + i);
      unrot_pair(g[2 * i], g[2 * i + 1], cs.x, cs.y, g[2 * i], g[2 * i + 1]);
    }
  }
}

// P = exp2(score * scale_log2 - lse2) and dS = P (dP - Delta) of 32 columns,
// packed to bf16 pairs (P only when WITH_P): nl and nd hold -lse2 and -Delta
// per column (kernel A, nstride 1) or one value for the whole row (kernel B,
// nstride 0); allowed(c) masks a column.
template <bool MASK, bool WITH_P, typename Allowed>
__device__ __forceinline__ void bwd_p_ds(const uint32_t (&sv)[32], const uint32_t (&dv)[32], const float* nl,
                                         const float* nd, int nstride, float sl2, Allowed allowed,
                                         uint32_t (&pk)[16], uint32_t (&dk)[16]) {
  const float2 sl22 = make_float2(sl2, sl2);
#pragma unroll
  for (int c = 0; c < 32; c += 2) {
    const float2 x = __ffma2_rn(make_float2(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])), sl22,
                                make_float2(nl[c * nstride], nl[(c + 1) * nstride]));
    float2 pv = make_float2(ex2(x.x), ex2(x.y));
    const float2 dd = __fadd2_rn(make_float2(__uint_as_float(dv[c]), __uint_as_float(dv[c + 1])),
                                 make_float2(nd[c * nstride], nd[(c + 1) * nstride]));
    float2 ds = __fmul2_rn(pv, dd);
    if constexpr (MASK) {
      // masked columns may hold stale values: select, never multiply
      if (!allowed(c)) pv.x = ds.x = 0.f;
      if (!allowed(c + 1)) pv.y = ds.y = 0.f;
    }
    if constexpr (WITH_P) pk[c >> 1] = pack_bf16x2(pv.x, pv.y);
    dk[c >> 1] = pack_bf16x2(ds.x, ds.y);
  }
}

// 1-D bulk copy global -> shared (16-byte aligned, size a multiple of 16),
// completing transaction bytes on `bar`.
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(smem_dst)),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// ---------------------------------------------------------------------------
// -Delta_t = -dO_t . O_t and minus the log-sum-exp in log2 units, one warp per row
// ---------------------------------------------------------------------------
struct BwdPrepArgs {
  const __nv_bfloat16* dout;   // [B, S, Hq, D]
  const float* out;            // [B, S, Hq, D]
  const float* lse;            // [B, Hq, S] natural log
  float* ndelta;               // [B, Hq, Sp] -Delta
  float* nlse2;                // [B, Hq, Sp] -lse * log2(e)
  int B, S, Hq, D, Sp;
};

__global__ void __launch_bounds__(256) bwd_prep_kernel(const BwdPrepArgs a) {
  const long long row = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long long nrows = static_cast<long long>(a.B) * a.S * a.Hq;
  if (row >= nrows) return;
  const int h = static_cast<int>(row % a.Hq);
  const long long bt = row / a.Hq;
  const int t = static_cast<int>(bt % a.S);
  const int b = static_cast<int>(bt / a.S);
  const __nv_bfloat16* g = a.dout + row * a.D;
  const float* o = a.out + row * a.D;
  float acc = 0.f;
  for (int d = lane * 2; d < a.D; d += 64) {
    const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(g + d));
    const float2 ov = __ldg(reinterpret_cast<const float2*>(o + d));
    acc = fmaf(bf16lo(w), ov.x, acc);
    acc = fmaf(bf16hi(w), ov.y, acc);
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) {
    const size_t i = (static_cast<size_t>(b) * a.Hq + h) * a.Sp + t;
    a.ndelta[i] = -acc;
    a.nlse2[i] = -__ldg(a.lse + (static_cast<size_t>(b) * a.Hq + h) * a.S + t) * 1.4426950408889634074f;
  }
}

// ---------------------------------------------------------------------------
// dK, dV: one CTA per 128-key tile of one (batch, kv head)
// ---------------------------------------------------------------------------
template <int D>
struct BwdKVSmem {
  static constexpr int kSlots = D == 128 ? 3 : 6;
  static constexpr int kKTile = kBM * D * 2;               // 128 keys
  static constexpr int kQTile = kBwdN * D * 2;             // 64 query rows
  static constexpr int kK0 = 0, kK1 = kKTile, kV = 2 * kKTile;
  static constexpr int kRing = 3 * kKTile;                 // [slot]{Q tile, dO tile}
  static constexpr int kSlotBytes = 2 * kQTile;
  static constexpr int kLD = kRing + kSlots * kSlotBytes;  // [slot]{lse2[64], delta[64]}
  static constexpr int kBar = kLD + kSlots * 2 * kBwdN * 4;
  // S^T/dP^T buffer sets in TMEM: three where they fit beside dV and dK
  // (D = 64: 3 x 64 + 3 x 64 + 2 x 64 = 512 columns), else two
  static constexpr int kBufs = 2 * 3 * kBwdN + 2 * D <= 512 ? 3 : 2;
  // kv_full, ring_full[S], ring_empty[S], s_full[B], dp_full[B], p_full[B], sd_free[B], dk_free,
  // s_free[B]
  static constexpr int kNumBars = 2 + 2 * kSlots + 5 * kBufs + 1;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kTotal = kMisc + 16;
  static constexpr int kAlloc = kTotal + 1024;
  static_assert(kAlloc <= 227 * 1024, "shared memory");
};

struct BwdKVPass {
  int j_lo, j_hi;     // 64-row query tiles
  int lo, hi;         // band hi <= t - s <= lo
  int sel;            // map
};

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ0, const __grid_constant__ CUtensorMap tmQ1,
                    const __grid_constant__ CUtensorMap tmK0, const __grid_constant__ CUtensorMap tmK1,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                    const BwdParams p) {
  using L = BwdKVSmem<D>;
  constexpr int NS = L::kSlots;
  constexpr int NB = L::kBufs;
  static_assert(2 * NB * kBwdN + 2 * D <= 512, "TMEM columns");
  constexpr int kCB = D / 64;
  constexpr uint32_t kIdescS = idesc_bf16_f32(kBM, kBwdN, false);   // keys x 64 queries
  constexpr uint32_t kIdescG = idesc_bf16_f32(kBM, D, true);        // keys x D, B MN-major

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* kv_full = bars;
  uint64_t* ring_full = bars + 1;
  uint64_t* ring_empty = ring_full + NS;
  uint64_t* s_full = ring_empty + NS;
  uint64_t* dp_full = s_full + NB;
  uint64_t* p_full = dp_full + NB;
  uint64_t* sd_free = p_full + NB;
  uint64_t* dk_free = sd_free + NB;
  uint64_t* s_free = dk_free + 1;   // the dV MMAs of the buffer's step are done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int grp = p.Hq / p.Hkv;
  // kv-head-major, the longest key tiles (the first ones) first
  const int kt = static_cast<int>(blockIdx.x) % p.nkt;
  const int bh = static_cast<int>(blockIdx.x) / p.nkt;
  const int hk = bh % p.Hkv, b = bh / p.Hkv;
  const int s0 = kt * kBM;
  const int s_last = min(p.S - 1, s0 + kBM - 1);

  BwdKVPass passes[2];
  int npass = 0;
  {
    int bands[2][3];
    const int nb = bwd_bands(p, bands);
    for (int i = 0; i < nb; ++i) {
      const long long t_min = static_cast<long long>(s0) + bands[i][1];
      const long long t_max =
          bands[i][0] >= kInf ? p.S - 1 : min(static_cast<long long>(p.S - 1), static_cast<long long>(s_last) + bands[i][0]);
      if (t_min > t_max) continue;
      passes[npass].j_lo = static_cast<int>(t_min / kBwdN);
      passes[npass].j_hi = static_cast<int>(t_max / kBwdN);
      passes[npass].lo = bands[i][0];
      passes[npass].hi = bands[i][1];
      passes[npass].sel = bands[i][2];
      ++npass;
    }
  }
  const bool two_maps = p.kind == kBifocal;

  if (tid == 0) {
    mbar_init(kv_full, 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(ring_full + i, 1);
      mbar_init(ring_empty + i, 1);
    }
    for (int a = 0; a < NB; ++a) {
      mbar_init(s_full + a, 1);
      mbar_init(dp_full + a, 1);
      mbar_init(p_full + a, 2 * kBM);
      mbar_init(sd_free + a, 1);
      mbar_init(s_free + a, 1);
    }
    mbar_init(dk_free, 2 * kBM);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tDP = tmem + NB * kBwdN, tDV = tmem + 2 * NB * kBwdN, tDK = tDV + D;

  if (warp == kBwdWarpTMA) {
    // ------------------------------------------------------------------ TMA
    if (lane == 0) {
      mbar_arrive_expect_tx(kv_full, (two_maps ? 3 : 2) * L::kKTile);
      for (int cb = 0; cb < kCB; ++cb) {
        tma_load_4d(smem + L::kK0 + cb * kBM * 128, &tmK0, kv_full, cb * 64, hk, s0, b);
        if (two_maps) tma_load_4d(smem + L::kK1 + cb * kBM * 128, &tmK1, kv_full, cb * 64, hk, s0, b);
        tma_load_4d(smem + L::kV + cb * kBM * 128, &tmV, kv_full, cb * 64, hk, s0, b);
      }
      int g = 0;
      bool ok = true;
      for (int pi = 0; pi < npass && ok; ++pi) {
        const CUtensorMap* tq = passes[pi].sel ? &tmQ1 : &tmQ0;
        for (int hh = 0; hh < grp && ok; ++hh) {
          const int h = hk * grp + hh;
          for (int j = passes[pi].j_lo; j <= passes[pi].j_hi; ++j, ++g) {
            const int slot = g % NS;
            if (g >= NS && !mbar_wait(ring_empty + slot, ((g / NS) - 1) & 1, abort_flag)) { ok = false; break; }
            uint8_t* dst = smem + L::kRing + slot * L::kSlotBytes;
            const int t0 = j * kBwdN;
            const int nv = min(kBwdN, p.S - t0);
            const uint32_t ldb = static_cast<uint32_t>(((nv * 4 + 15) / 16) * 16);
            mbar_arrive_expect_tx(ring_full + slot, 2 * L::kQTile + 2 * ldb);
            for (int cb = 0; cb < kCB; ++cb) {
              tma_load_4d(dst + cb * kBwdN * 128, tq, ring_full + slot, cb * 64, h, t0, b);
              tma_load_4d(dst + L::kQTile + cb * kBwdN * 128, &tmDO, ring_full + slot, cb * 64, h, t0, b);
            }
            float* ld = reinterpret_cast<float*>(smem + L::kLD) + slot * 2 * kBwdN;
            const size_t row = (static_cast<size_t>(b) * p.Hq + h) * p.Sp + t0;
            bulk_load(ld, p.nlse2 + row, ldb, ring_full + slot);
            bulk_load(ld + kBwdN, p.ndelta + row, ldb, ring_full + slot);
          }
        }
      }
    }
  } else if (warp == kBwdWarpS || warp == kBwdWarpDP) {
    // ------------------------------------- MMA: S^T = K_r Q_r^T, dP^T = V dO^T
    if (lane == 0) {
      const bool is_s = warp == kBwdWarpS;
      uint64_t* done = is_s ? s_full : dp_full;
      const uint32_t dcol = is_s ? tS : tDP;
      bool ok = mbar_wait(kv_full, 0, abort_flag);
      int g = 0;
      for (int pi = 0; pi < npass && ok; ++pi) {
        const uint32_t aaddr = smem_u32(smem + (is_s ? (passes[pi].sel ? L::kK1 : L::kK0) : L::kV));
        const int T = passes[pi].j_hi - passes[pi].j_lo + 1;
        for (int step = 0; step < grp * T; ++step, ++g) {
          const int slot = g % NS, buf = g % NB;
          if (!mbar_wait(ring_full + slot, (g / NS) & 1, abort_flag)) { ok = false; break; }
          // the buffer's P^T (S^T side) or dS^T (dP^T side) of step g - NB has
          // been read by its dV or dK MMAs; S^T is queued behind the dK MMAs
          if (g >= NB && !mbar_wait((is_s ? s_free : sd_free) + buf, ((g / NB) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t baddr = smem_u32(smem + L::kRing + slot * L::kSlotBytes + (is_s ? 0 : L::kQTile));
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t kin = (kk & 3) * 32;
            umma_ss(dcol + buf * kBwdN, sdesc_sw128(aaddr + (kk >> 2) * kBM * 128 + kin, 16, 1024),
                    sdesc_sw128(baddr + (kk >> 2) * kBwdN * 128 + kin, 16, 1024), kIdescS, kk > 0 ? 1u : 0u);
          }
          umma_commit(done + buf);
        }
      }
    }
  } else if (warp == kBwdWarpG) {
    // ------------------------------ MMA: dV += P^T dO, dK += dS^T Q_r (A from TMEM)
    if (lane == 0) {
      int g = 0;
      bool ok = true;
      for (int pi = 0; pi < npass && ok; ++pi) {
        const int T = passes[pi].j_hi - passes[pi].j_lo + 1;
        for (int step = 0; step < grp * T; ++step, ++g) {
          const int slot = g % NS, buf = g % NB;
          if (!mbar_wait(p_full + buf, (g / NB) & 1, abort_flag)) { ok = false; break; }
          // the previous pass's dK has been read out (parked) before it is reset
          if (step == 0 && pi > 0 && !mbar_wait(dk_free, (pi - 1) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t qaddr = smem_u32(smem + L::kRing + slot * L::kSlotBytes);
          const uint32_t oaddr = qaddr + L::kQTile;
#pragma unroll
          for (int kk = 0; kk < kBwdN / 16; ++kk) {
            umma_ts(tDV, tS + buf * kBwdN + bwd_pcol(kk), sdesc_sw128(oaddr + kk * 2048, kBwdN * 128, 1024),
                    kIdescG, (g > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(s_free + buf);
#pragma unroll
          for (int kk = 0; kk < kBwdN / 16; ++kk) {
            umma_ts(tDK, tDP + buf * kBwdN + bwd_pcol(kk), sdesc_sw128(qaddr + kk * 2048, kBwdN * 128, 1024),
                    kIdescG, (step > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(sd_free + buf);
          umma_commit(ring_empty + slot);
        }
      }
    }
  } else if (warp < 8) {
    // ----------------------------------------------- softmax side, epilogue
    const int r = tid & (kBM - 1);           // key row in the tile = TMEM lane
    const int hw = warp >> 2;                // warpgroup: columns [32 hw, 32 hw + 32)
    const int s = s0 + r;
    const bool row_ok = s < p.S;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
    };
    const float sl2 = p.scale_log2;
    bool ok = true;
    int g = 0;
    for (int pi = 0; pi < npass && ok; ++pi) {
      const BwdKVPass ps = passes[pi];
      const int T = ps.j_hi - ps.j_lo + 1;
      for (int step = 0; step < grp * T; ++step, ++g) {
        const int slot = g % NS, buf = g % NB;
        const int j = ps.j_lo + step % T;
        if (!wwait(ring_full + slot, (g / NS) & 1) || !wwait(s_full + buf, (g / NB) & 1) ||
            !wwait(dp_full + buf, (g / NB) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t sv[32], dv[32];
        tmem_ld32(tS + buf * kBwdN + hw * 32 + lane_off, sv);
        tmem_ld32(tDP + buf * kBwdN + hw * 32 + lane_off, dv);
        tmem_ld_wait();
        const float* nl = reinterpret_cast<const float*>(smem + L::kLD) + slot * 2 * kBwdN + hw * 32;
        const int t0 = j * kBwdN + hw * 32;   // query row of this warpgroup's first column
        // every (t, s) pair of the tile is inside the band: no per-column test
        const bool full = (static_cast<long long>(j * kBwdN) - s_last >= ps.hi) &&
                          (static_cast<long long>(j * kBwdN + kBwdN - 1) - s0 <= ps.lo) &&
                          (j * kBwdN + kBwdN <= p.S) && (s0 + kBM <= p.S);
        uint32_t pk[16], dk2[16];
        if (full) {
          bwd_p_ds<false, true>(sv, dv, nl, nl + kBwdN, 1, sl2, [](int) { return true; }, pk, dk2);
        } else {
          auto allowed = [&](int c) {
            const int dd = t0 + c - s;
            return row_ok && t0 + c < p.S && dd >= ps.hi && dd <= ps.lo;
          };
          bwd_p_ds<true, true>(sv, dv, nl, nl + kBwdN, 1, sl2, allowed, pk, dk2);
        }
        // P^T and dS^T (bf16) over the first 16 of this warpgroup's columns
        tmem_st16(tS + buf * kBwdN + hw * 32 + lane_off, pk);
        tmem_st16(tDP + buf * kBwdN + hw * 32 + lane_off, dk2);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(p_full + buf);
      }
      if (!ok) break;
      // ---- pass epilogue: dK of this map, turned back and scaled; this
      // warpgroup's half of the columns
      if (!wwait(sd_free + ((g - 1) % NB), ((g - 1) / NB) & 1)) { ok = false; break; }
      tc_fence_after();
      float gk[D / 2];
      const float2* tab = p.tab0 == nullptr ? nullptr
                          : (ps.sel ? p.tab1 : p.tab0) + static_cast<size_t>(row_ok ? s : 0) * (D / 2);
      grad_half_from_tmem<D>(tDK + lane_off, p.scale, tab, hw * (D / 2), gk);
      tc_fence_before();
      if (pi + 1 < npass) mbar_arrive(dk_free);   // the next pass may reset dK
      if (row_ok) {
        float* dst = p.dk + ((static_cast<size_t>(b) * p.S + s) * p.Hkv + hk) * D;
        store_grad_half<D>(dst, gk, hw * (D / 2), two_maps && pi > 0, p.half != 0);
      }
    }
    // ---- dV (every pass and head), after the last gradient MMA
    if (ok && g > 0 && wwait(sd_free + ((g - 1) % NB), ((g - 1) / NB) & 1)) {
      tc_fence_after();
      float gv[D / 2];
      grad_half_from_tmem<D>(tDV + lane_off, 1.0f, nullptr, hw * (D / 2), gv);
      if (row_ok) {
        float* dst = p.dv + ((static_cast<size_t>(b) * p.S + s) * p.Hkv + hk) * D;
        store_grad_half<D>(dst, gv, hw * (D / 2), false, false);
      }
    } else if (ok && g == 0 && row_ok) {
      // a key no query attends (not reached for causal bands, kept for safety)
      float* dst = p.dv + ((static_cast<size_t>(b) * p.S + s) * p.Hkv + hk) * D;
      float* dstk = p.dk + ((static_cast<size_t>(b) * p.S + s) * p.Hkv + hk) * D;
      for (int e = hw * (D / 2); e < (hw + 1) * (D / 2); ++e) dst[e] = dstk[e] = 0.f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    const unsigned long long t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 20000000ull) __nanosleep(100000);
  }
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// dQ: one CTA per 128-row query tile of one (batch, query head)
// ---------------------------------------------------------------------------
template <int D>
struct BwdQSmem {
  static constexpr int kSlots = D == 128 ? 4 : 8;
  static constexpr int kQTile = kBM * D * 2;               // 128 query rows
  static constexpr int kKTile = kBwdN * D * 2;             // 64 keys
  static constexpr int kQ = 0, kDO = kQTile;
  static constexpr int kRing = 2 * kQTile;                 // [slot]{K tile, V tile}
  static constexpr int kSlotBytes = 2 * kKTile;
  static constexpr int kBar = kRing + kSlots * kSlotBytes;
  // S/dP buffer sets in TMEM: three (S 3 x 64, dP 3 x 64 and dQ D columns fit
  // in 512), so the chain S -> dS -> dQ MMA of one set spans three tiles
  static constexpr int kBufs = 3;
  // q_full, q_free, dq_free, ring_full[S], ring_empty[S], s_full[B], dp_full[B], p_full[B], sd_free[B]
  static constexpr int kNumBars = 3 + 2 * kSlots + 4 * kBufs;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kTotal = kMisc + 16;
  static constexpr int kAlloc = kTotal + 1024;
  static_assert(kAlloc <= 227 * 1024, "shared memory");
};

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ0, const __grid_constant__ CUtensorMap tmQ1,
                  const __grid_constant__ CUtensorMap tmK0, const __grid_constant__ CUtensorMap tmK1,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                  const BwdParams p) {
  using L = BwdQSmem<D>;
  constexpr int NS = L::kSlots;
  constexpr int NB = L::kBufs;
  constexpr int kCB = D / 64;
  static_assert(2 * NB * kBwdN + D <= 512, "TMEM columns");
  constexpr uint32_t kIdescS = idesc_bf16_f32(kBM, kBwdN, false);   // queries x 64 keys
  constexpr uint32_t kIdescG = idesc_bf16_f32(kBM, D, true);        // queries x D, B MN-major

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* q_full = bars;
  uint64_t* q_free = bars + 1;
  uint64_t* dq_free = bars + 2;
  uint64_t* ring_full = bars + 3;
  uint64_t* ring_empty = ring_full + NS;
  uint64_t* s_full = ring_empty + NS;
  uint64_t* dp_full = s_full + NB;
  uint64_t* p_full = dp_full + NB;
  uint64_t* sd_free = p_full + NB;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int grp = p.Hq / p.Hkv;
  // kv-head-major: all query tiles (longest first) and heads of one (batch,
  // kv head) before the next, so resident CTAs share the key/value tiles in L2
  const int per_kv = p.nqt * grp;
  const int bhk = static_cast<int>(blockIdx.x) / per_kv;
  const int r2 = static_cast<int>(blockIdx.x) % per_kv;
  const int b = bhk / p.Hkv, hk = bhk % p.Hkv;
  const int qt = p.nqt - 1 - r2 / grp;
  const int h = hk * grp + r2 % grp;
  const int t0 = qt * kBM;
  const int t_last = min(p.S - 1, t0 + kBM - 1);

  BwdKVPass passes[2];   // here: 64-key tiles [j_lo, j_hi]
  int npass = 0;
  {
    int bands[2][3];
    const int nb = bwd_bands(p, bands);
    for (int i = 0; i < nb; ++i) {
      const long long s_min = bands[i][0] >= kInf ? 0 : max(0LL, static_cast<long long>(t0) - bands[i][0]);
      const long long s_max = min(static_cast<long long>(p.S - 1), static_cast<long long>(t_last) - bands[i][1]);
      if (s_max < s_min) continue;
      passes[npass].j_lo = static_cast<int>(s_min / kBwdN);
      passes[npass].j_hi = static_cast<int>(s_max / kBwdN);
      passes[npass].lo = bands[i][0];
      passes[npass].hi = bands[i][1];
      passes[npass].sel = bands[i][2];
      ++npass;
    }
  }
  const bool two_maps = p.kind == kBifocal;

  if (tid == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_free, 1);
    mbar_init(dq_free, 2 * kBM);
    for (int i = 0; i < NS; ++i) {
      mbar_init(ring_full + i, 1);
      mbar_init(ring_empty + i, 1);
    }
    for (int a = 0; a < NB; ++a) {
      mbar_init(s_full + a, 1);
      mbar_init(dp_full + a, 1);
      mbar_init(p_full + a, 2 * kBM);
      mbar_init(sd_free + a, 1);
    }
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tDP = tmem + NB * kBwdN, tDQ = tmem + 2 * NB * kBwdN;

  if (warp == kBwdWarpTMA) {
    // ------------------------------------------------------------------ TMA
    if (lane == 0) {
      int g = 0;
      bool ok = true;
      for (int pi = 0; pi < npass && ok; ++pi) {
        // the query and dO tiles of the previous pass are no longer read
        if (pi > 0 && !mbar_wait(q_free, (pi - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(q_full, 2 * L::kQTile);
        const CUtensorMap* tq = passes[pi].sel ? &tmQ1 : &tmQ0;
        for (int cb = 0; cb < kCB; ++cb) {
          tma_load_4d(smem + L::kQ + cb * kBM * 128, tq, q_full, cb * 64, h, t0, b);
          tma_load_4d(smem + L::kDO + cb * kBM * 128, &tmDO, q_full, cb * 64, h, t0, b);
        }
        const CUtensorMap* tk = passes[pi].sel ? &tmK1 : &tmK0;
        for (int j = passes[pi].j_lo; j <= passes[pi].j_hi; ++j, ++g) {
          const int slot = g % NS;
          if (g >= NS && !mbar_wait(ring_empty + slot, ((g / NS) - 1) & 1, abort_flag)) { ok = false; break; }
          uint8_t* dst = smem + L::kRing + slot * L::kSlotBytes;
          mbar_arrive_expect_tx(ring_full + slot, L::kSlotBytes);
          for (int cb = 0; cb < kCB; ++cb) {
            tma_load_4d(dst + cb * kBwdN * 128, tk, ring_full + slot, cb * 64, hk, j * kBwdN, b);
            tma_load_4d(dst + L::kKTile + cb * kBwdN * 128, &tmV, ring_full + slot, cb * 64, hk, j * kBwdN, b);
          }
        }
      }
    }
  } else if (warp == kBwdWarpS || warp == kBwdWarpDP) {
    // ----------------------------------------- MMA: S = Q_r K_r^T, dP = dO V^T
    if (lane == 0) {
      const bool is_s = warp == kBwdWarpS;
      uint64_t* done = is_s ? s_full : dp_full;
      const uint32_t dcol = is_s ? tS : tDP;
      const uint32_t aaddr = smem_u32(smem + (is_s ? L::kQ : L::kDO));
      int g = 0;
      bool ok = true;
      for (int pi = 0; pi < npass && ok; ++pi) {
        if (!mbar_wait(q_full, pi & 1, abort_flag)) break;
        const int T = passes[pi].j_hi - passes[pi].j_lo + 1;
        for (int step = 0; step < T; ++step, ++g) {
          const int slot = g % NS, buf = g % NB;
          if (!mbar_wait(ring_full + slot, (g / NS) & 1, abort_flag)) { ok = false; break; }
          if (g >= NB && !mbar_wait(sd_free + buf, ((g / NB) - 1) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t baddr = smem_u32(smem + L::kRing + slot * L::kSlotBytes + (is_s ? 0 : L::kKTile));
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t kin = (kk & 3) * 32;
            umma_ss(dcol + buf * kBwdN, sdesc_sw128(aaddr + (kk >> 2) * kBM * 128 + kin, 16, 1024),
                    sdesc_sw128(baddr + (kk >> 2) * kBwdN * 128 + kin, 16, 1024), kIdescS, kk > 0 ? 1u : 0u);
          }
          umma_commit(done + buf);
        }
      }
    }
  } else if (warp == kBwdWarpG) {
    // ------------------------------------------ MMA: dQ += dS K_r (A from TMEM)
    if (lane == 0) {
      int g = 0;
      bool ok = true;
      for (int pi = 0; pi < npass && ok; ++pi) {
        const int T = passes[pi].j_hi - passes[pi].j_lo + 1;
        for (int step = 0; step < T; ++step, ++g) {
          const int slot = g % NS, buf = g % NB;
          if (!mbar_wait(p_full + buf, (g / NB) & 1, abort_flag)) { ok = false; break; }
          if (step == 0 && pi > 0 && !mbar_wait(dq_free, (pi - 1) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t kaddr = smem_u32(smem + L::kRing + slot * L::kSlotBytes);
#pragma unroll
          for (int kk = 0; kk < kBwdN / 16; ++kk) {
            umma_ts(tDQ, tS + buf * kBwdN + bwd_pcol(kk), sdesc_sw128(kaddr + kk * 2048, kBwdN * 128, 1024),
                    kIdescG, (step > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(sd_free + buf);
          umma_commit(ring_empty + slot);
          if (step == T - 1 && pi + 1 < npass) umma_commit(q_free);
        }
      }
    }
  } else if (warp < 8) {
    // ----------------------------------------------- softmax side, epilogue
    const int r = tid & (kBM - 1);           // query row in the tile = TMEM lane
    const int hw = warp >> 2;                // warpgroup: key columns [32 hw, 32 hw + 32)
    const int t = t0 + r;
    const bool row_ok = t < p.S;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
    };
    const float sl2 = p.scale_log2;
    const size_t lrow = (static_cast<size_t>(b) * p.Hq + h) * p.Sp + (row_ok ? t : 0);
    const float nl = __ldg(p.nlse2 + lrow);
    const float nd = __ldg(p.ndelta + lrow);
    float* dst = p.dq + ((static_cast<size_t>(b) * p.S + (row_ok ? t : 0)) * p.Hq + h) * D;
    bool ok = true;
    int g = 0;
    for (int pi = 0; pi < npass && ok; ++pi) {
      const BwdKVPass ps = passes[pi];
      const int T = ps.j_hi - ps.j_lo + 1;
      for (int step = 0; step < T; ++step, ++g) {
        const int buf = g % NB;
        const int kv0 = (ps.j_lo + step) * kBwdN;
        if (!wwait(s_full + buf, (g / NB) & 1) || !wwait(dp_full + buf, (g / NB) & 1)) { ok = false; break; }
        tc_fence_after();
        uint32_t sv[32], dv[32];
        tmem_ld32(tS + buf * kBwdN + hw * 32 + lane_off, sv);
        tmem_ld32(tDP + buf * kBwdN + hw * 32 + lane_off, dv);
        tmem_ld_wait();
        const bool full = (static_cast<long long>(t0) - (kv0 + kBwdN - 1) >= ps.hi) &&
                          (static_cast<long long>(t_last) - kv0 <= ps.lo) && (t0 + kBM <= p.S) &&
                          (kv0 + kBwdN <= p.S);
        const int k0 = kv0 + hw * 32;        // key of this warpgroup's first column
        uint32_t pk[16], dk2[16];
        if (full) {
          bwd_p_ds<false, false>(sv, dv, &nl, &nd, 0, sl2, [](int) { return true; }, pk, dk2);
        } else {
          auto allowed = [&](int c) {
            const int dd = t - (k0 + c);
            return row_ok && k0 + c < p.S && dd >= ps.hi && dd <= ps.lo;
          };
          bwd_p_ds<true, false>(sv, dv, &nl, &nd, 0, sl2, allowed, pk, dk2);
        }
        tmem_st16(tS + buf * kBwdN + hw * 32 + lane_off, dk2);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(p_full + buf);
      }
      if (!ok) break;
      // ---- pass epilogue: dQ of this map, turned back and scaled; this
      // warpgroup's half of the columns
      if (!wwait(sd_free + ((g - 1) % NB), ((g - 1) / NB) & 1)) { ok = false; break; }
      tc_fence_after();
      float gq[D / 2];
      const float2* tab = p.tab0 == nullptr ? nullptr
                          : (ps.sel ? p.tab1 : p.tab0) + static_cast<size_t>(row_ok ? t : 0) * (D / 2);
      grad_half_from_tmem<D>(tDQ + lane_off, p.scale, tab, hw * (D / 2), gq);
      tc_fence_before();
      if (pi + 1 < npass) mbar_arrive(dq_free);
      if (row_ok) store_grad_half<D>(dst, gq, hw * (D / 2), two_maps && pi > 0, p.half != 0);
    }
    if (ok && npass == 0 && row_ok) {
      for (int e = hw * (D / 2); e < (hw + 1) * (D / 2); ++e) dst[e] = 0.f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    const unsigned long long t0n = globaltimer_ns();
    while (globaltimer_ns() - t0n < 20000000ull) __nanosleep(100000);
  }
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace ropeattn
