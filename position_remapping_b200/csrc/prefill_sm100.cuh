// Causal prefill attention with RoPE at remapped positions, sm_100a.
//
// One CTA computes one 128-row query tile of one (batch, query head):
//   warps 0-3  softmax: rotate the staged query tile in shared memory, then
//              for every key tile read S = Q K^T from TMEM (one row per
//              thread), mask, online softmax in the exp2 domain, write P
//              (bf16) back over S in TMEM, and finally normalise, merge and
//              store O and the log-sum-exp.
//   warp 4     TMA producer: query tile once, then key/value tiles through an
//              NST-stage ring (128-byte swizzle, no multicast).
//   warp 5     MMA issuer (one thread): S = Q K^T (SS form) and O += P V (TS
//              form, P read from TMEM) with fp32 accumulators in TMEM.
// TMEM: S/P double buffer in columns [0, 256), O accumulators from 256
// (O[0] main/local, O[1] remote).
//
// A pass is a sweep over key tiles with one query operand, one key tensor, a
// distance band hi_off <= t - s <= lo_off, and one accumulator:
//   standard / EndPrompt / NoPE: one pass, band [0, inf) (causal);
//   Periodic RoPE: one pass, band [0, W-1] (the window {t-W+1..t}, §3.2);
//   Jet-Long bifocal: a remote pass, band [w0+1, inf), with the remote query
//   and keys, then a local pass, band [0, w0], with the exact ones (Eq. 1).
// The bifocal passes are the remote-only term W_B O_B - W_C O_C and the call-A
// term of the inclusion-exclusion merge (Jet-Long §3.3 Eq. 7), obtained by
// masking instead of subtraction; the epilogue merges them by their
// log-sum-exp in fp32.
#pragma once

#include "common.cuh"
#include "posmap.cuh"

namespace ropeattn {

constexpr int kBM = 128;  // query rows per tile (TMEM lanes)
constexpr int kBN = 128;  // keys per tile
constexpr int kPrefillThreads = 192;
constexpr int kInf = 0x3fffffff;

struct PrefillParams {
  float* out;          // [B, S, Hq, D]
  float* lse;          // [B, Hq, S]
  const float2* tab0;  // [S][D/2] query (cos, sin) at map-0 positions (null for NoPE)
  const float2* tab1;  // [S][D/2] at remote positions (bifocal)
  int B, S, Hq, Hkv;
  int nqt;             // query tiles per (b, h)
  int kind;
  int window;          // Periodic RoPE
  int w0;              // Jet-Long
  float scale_log2;    // softmax scale * log2(e)
};

struct PassDesc {
  int j_lo, j_hi;      // key tiles [j_lo, j_hi]
  int lo_off, hi_off;  // allowed band: hi_off <= t - s <= lo_off
  int sel;             // 0: Q0/K0/O0 (main or local), 1: Q1/K1/O1 (remote)
};

__device__ __forceinline__ int make_passes(const PrefillParams& p, int q0, PassDesc* ps) {
  int bands[2][3];  // lo_off, hi_off, sel
  int nb = 0;
  if (p.kind == kBifocal) {
    bands[0][0] = kInf; bands[0][1] = p.w0 + 1; bands[0][2] = 1;
    bands[1][0] = p.w0; bands[1][1] = 0; bands[1][2] = 0;
    nb = 2;
  } else if (p.kind == kPeriodic) {
    bands[0][0] = p.window - 1; bands[0][1] = 0; bands[0][2] = 0;
    nb = 1;
  } else {
    bands[0][0] = kInf; bands[0][1] = 0; bands[0][2] = 0;
    nb = 1;
  }
  int n = 0;
  for (int i = 0; i < nb; ++i) {
    const int lo_off = bands[i][0], hi_off = bands[i][1];
    int s_min = lo_off >= kInf ? 0 : max(0, q0 - lo_off);
    int s_max = min(p.S - 1, q0 + kBM - 1 - hi_off);
    if (s_max < s_min) continue;
    ps[n].j_lo = s_min / kBN;
    ps[n].j_hi = s_max / kBN;
    ps[n].lo_off = lo_off;
    ps[n].hi_off = hi_off;
    ps[n].sel = bands[i][2];
    ++n;
  }
  return n;
}

template <int D, int NST>
struct PrefillSmem {
  static constexpr int kQBytes = kBM * D * 2;
  static constexpr int kKVBytes = kBN * D * 2;
  static constexpr int kQ0 = 0;
  static constexpr int kQ1 = kQ0 + kQBytes;
  static constexpr int kK = kQ1 + kQBytes;
  static constexpr int kV = kK + NST * kKVBytes;
  static constexpr int kBar = kV + NST * kKVBytes;
  // barriers: q_full, q_ready, k_full[NST], k_empty[NST], v_full[NST],
  // v_empty[NST], s_full[2], p_full[2], o_done, o_final
  static constexpr int kNumBars = 2 + 4 * NST + 6;
  static constexpr int kMisc = kBar + kNumBars * 8;  // tmem base (u32), abort flag (int)
  static constexpr int kTotal = kMisc + 16;
  static constexpr int kAlloc = kTotal + 1024;       // slack to align the base to 1024
};

template <int D, int NST>
__global__ void __launch_bounds__(kPrefillThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK0,
                   const __grid_constant__ CUtensorMap tmK1, const __grid_constant__ CUtensorMap tmV,
                   const PrefillParams p) {
  using L = PrefillSmem<D, NST>;
  constexpr int kCB = D / 64;              // 64-column (128-byte) swizzle blocks per row
  constexpr int kBlockBytes = kBM * 128;   // one swizzle block of a 128-row tile
  constexpr uint32_t kIdescQK = idesc_bf16_f32(kBM, kBN, false);
  constexpr uint32_t kIdescPV = idesc_bf16_f32(kBM, D, true);
  constexpr uint32_t kTmemCols = 512;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ0 = smem + L::kQ0;
  uint8_t* sQ1 = smem + L::kQ1;
  uint8_t* sK = smem + L::kK;
  uint8_t* sV = smem + L::kV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* q_full = bars + 0;
  uint64_t* q_ready = bars + 1;
  uint64_t* k_full = bars + 2;
  uint64_t* k_empty = k_full + NST;
  uint64_t* v_full = k_empty + NST;
  uint64_t* v_empty = v_full + NST;
  uint64_t* s_full = v_empty + NST;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_done = p_full + 2;   // one arrival per PV (rescale waits)
  uint64_t* o_final = o_done + 1;  // one arrival after the last PV (epilogue)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  // work item: longest (last) query tiles first; heads of one tile adjacent
  const int per_tile = p.Hq * p.B;
  const int qt = p.nqt - 1 - static_cast<int>(blockIdx.x) / per_tile;
  const int rem = static_cast<int>(blockIdx.x) % per_tile;
  const int h = rem % p.Hq;
  const int b = rem / p.Hq;
  const int hk = h / (p.Hq / p.Hkv);
  const int q0 = qt * kBM;

  PassDesc passes[2];
  const int npass = make_passes(p, q0, passes);

  if (tid == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_ready, kBM);
    for (int i = 0; i < NST; ++i) {
      mbar_init(k_full + i, 1);
      mbar_init(k_empty + i, 1);
      mbar_init(v_full + i, 1);
      mbar_init(v_empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full + i, 1);
      mbar_init(p_full + i, kBM);
    }
    mbar_init(o_done, 1);
    mbar_init(o_final, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK0);
    tma_prefetch_desc(&tmK1);
    tma_prefetch_desc(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem;            // S/P buffers at columns 0 and 128
  const uint32_t tO = tmem + 256;      // O[sel] at 256 + sel * D

  if (warp == 4) {
    // ------------------------------------------------------------------ TMA
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, L::kQBytes);
      for (int cb = 0; cb < kCB; ++cb) tma_load_4d(sQ0 + cb * kBlockBytes, &tmQ, q_full, cb * 64, h, q0, b);
      int g = 0;
      bool ok = true;
      for (int pi = 0; pi < npass && ok; ++pi) {
        const CUtensorMap* tk = passes[pi].sel ? &tmK1 : &tmK0;
        for (int j = passes[pi].j_lo; j <= passes[pi].j_hi; ++j, ++g) {
          const int st = g % NST;
          const uint32_t ph = (g / NST) & 1;
          if (!mbar_wait(k_empty + st, ph ^ 1, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(k_full + st, L::kKVBytes);
          for (int cb = 0; cb < kCB; ++cb)
            tma_load_4d(sK + st * L::kKVBytes + cb * kBlockBytes, tk, k_full + st, cb * 64, hk, j * kBN, b);
          if (!mbar_wait(v_empty + st, ph ^ 1, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(v_full + st, L::kKVBytes);
          for (int cb = 0; cb < kCB; ++cb)
            tma_load_4d(sV + st * L::kKVBytes + cb * kBlockBytes, &tmV, v_full + st, cb * 64, hk, j * kBN, b);
        }
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0) {
      bool ok = mbar_wait(q_ready, 0, abort_flag);
      tc_fence_after();
      int g = 0;
      int prev_sel = 0, prev_first = 1;
      auto issue_pv = [&](int x, int sel, int first) -> bool {
        const int sb = x & 1;
        if (!mbar_wait(p_full + sb, (x >> 1) & 1, abort_flag)) return false;
        const int st = x % NST;
        if (!mbar_wait(v_full + st, (x / NST) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t vaddr = smem_u32(sV + st * L::kKVBytes);
        const uint32_t d = tO + sel * D;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          const uint64_t bdesc = sdesc_sw128(vaddr + kk * 2048, kBlockBytes, 1024);
          umma_ts(d, tS + sb * 128 + kk * 8, bdesc, kIdescPV, (kk > 0 || !first) ? 1u : 0u);
        }
        umma_commit(v_empty + st);
        umma_commit(o_done);
        return true;
      };
      for (int pi = 0; pi < npass && ok; ++pi) {
        const int sel = passes[pi].sel;
        const uint32_t qaddr = smem_u32(sel ? sQ1 : sQ0);
        for (int j = passes[pi].j_lo; j <= passes[pi].j_hi && ok; ++j, ++g) {
          const int st = g % NST;
          if (!mbar_wait(k_full + st, (g / NST) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t kaddr = smem_u32(sK + st * L::kKVBytes);
          const uint32_t d = tS + (g & 1) * 128;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * kBlockBytes + (kk & 3) * 32;
            umma_ss(d, sdesc_sw128(qaddr + off, 16, 1024), sdesc_sw128(kaddr + off, 16, 1024), kIdescQK,
                    kk > 0 ? 1u : 0u);
          }
          umma_commit(s_full + (g & 1));
          umma_commit(k_empty + st);
          if (g > 0 && !issue_pv(g - 1, prev_sel, prev_first)) { ok = false; break; }
          prev_sel = sel;
          prev_first = (j == passes[pi].j_lo);
        }
      }
      if (ok && g > 0 && issue_pv(g - 1, prev_sel, prev_first)) umma_commit(o_final);
    }
  } else {
    // -------------------------------------------------------------- softmax
    const int row = tid;               // TMEM lane == query row in the tile
    const int t = q0 + row;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    // waits are made warp-uniform so the warp-collective TMEM accesses that
    // follow are always executed by all 32 lanes together
    auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
    };
    bool ok = wwait(q_full, 0);
    // rotate this row of the staged query tile (Periodic RoPE §3.1 Eq. 2 at
    // the kind's positions; bifocal also writes the remote-position copy)
    if (ok && p.tab0 != nullptr) {
      const bool bif = p.kind == kBifocal;
      const float4* tr0 = reinterpret_cast<const float4*>(p.tab0 + static_cast<size_t>(t) * (D / 2));
      const float4* tr1 = bif ? reinterpret_cast<const float4*>(p.tab1 + static_cast<size_t>(t) * (D / 2)) : nullptr;
#pragma unroll 4
      for (int c = 0; c < D / 8; ++c) {
        const int off = (c >> 3) * kBlockBytes + row * 128 + (((c & 7) ^ (row & 7)) << 4);
        uint4* src = reinterpret_cast<uint4*>(sQ0 + off);
        if (t < p.S) {
          const uint4 x = *src;
          const uint32_t xw[4] = {x.x, x.y, x.z, x.w};
          uint32_t y0[4], y1[4];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float4 cs0 = __ldg(tr0 + c * 2 + e);   // pairs 4c+2e, 4c+2e+1
            float a0, a1;
            rot_pair(bf16lo(xw[2 * e]), bf16hi(xw[2 * e]), cs0.x, cs0.y, a0, a1);
            y0[2 * e] = pack_bf16x2(a0, a1);
            rot_pair(bf16lo(xw[2 * e + 1]), bf16hi(xw[2 * e + 1]), cs0.z, cs0.w, a0, a1);
            y0[2 * e + 1] = pack_bf16x2(a0, a1);
            if (bif) {
              const float4 cs1 = __ldg(tr1 + c * 2 + e);
              rot_pair(bf16lo(xw[2 * e]), bf16hi(xw[2 * e]), cs1.x, cs1.y, a0, a1);
              y1[2 * e] = pack_bf16x2(a0, a1);
              rot_pair(bf16lo(xw[2 * e + 1]), bf16hi(xw[2 * e + 1]), cs1.z, cs1.w, a0, a1);
              y1[2 * e + 1] = pack_bf16x2(a0, a1);
            }
          }
          *src = make_uint4(y0[0], y0[1], y0[2], y0[3]);
          if (bif) *reinterpret_cast<uint4*>(sQ1 + off) = make_uint4(y1[0], y1[1], y1[2], y1[3]);
        } else if (bif) {
          *reinterpret_cast<uint4*>(sQ1 + off) = make_uint4(0u, 0u, 0u, 0u);
        }
      }
    }
    fence_proxy_async_smem();
    mbar_arrive(q_ready);

    const float sl2 = p.scale_log2;
    float m_row[2] = {-INFINITY, -INFINITY};  // running max (log2 domain), per accumulator
    float l_row[2] = {0.f, 0.f};
    int g = 0;
    for (int pi = 0; pi < npass && ok; ++pi) {
      const PassDesc ps = passes[pi];
      float m = -INFINITY, l = 0.f;
      for (int j = ps.j_lo; j <= ps.j_hi; ++j, ++g) {
        const int sb = g & 1;
        if (!wwait(s_full + sb, (g >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        float s[kBN];
        {
          uint32_t r[32];
#pragma unroll
          for (int c = 0; c < kBN / 32; ++c) {
            tmem_ld32(tS + sb * 128 + c * 32 + lane_off, r);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) s[c * 32 + e] = __uint_as_float(r[e]);
          }
        }
        const int kv0 = j * kBN;
        const bool full = (q0 - kv0 - (kBN - 1) >= ps.hi_off) && (q0 + kBM - 1 - kv0 <= ps.lo_off);
        if (!full) {
          const int dbase = t - kv0;  // t - s = dbase - c
#pragma unroll
          for (int c = 0; c < kBN; ++c) {
            const int d = dbase - c;
            if (d < ps.hi_off || d > ps.lo_off) s[c] = -INFINITY;
          }
        }
        float mx8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) mx8[e] = s[e];
#pragma unroll
        for (int c = 8; c < kBN; c += 8)
#pragma unroll
          for (int e = 0; e < 8; ++e) mx8[e] = fmaxf(mx8[e], s[c + e]);
        float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                         fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
        mx *= sl2;
        // lazy rescale: move the reference max only when it grows by > 8 (x256)
        const bool need = mx > m + 8.0f;
        const float m_new = need ? mx : m;
        const float alpha = need ? ex2(m - m_new) : 1.0f;
        l *= alpha;
        if (j != ps.j_lo && __any_sync(0xffffffffu, need)) {
          // PV of the previous tile must be complete before O is rescaled
          if (!wwait(o_done, (g - 1) & 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t to = tO + ps.sel * D + lane_off;
          uint32_t r[32];
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            tmem_ld32(to + c * 32, r);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
            tmem_st32(to + c * 32, r);
          }
        }
        m = m_new;
        const float mu = (m == -INFINITY) ? 0.f : m;
        float l8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        uint32_t pk[kBN / 2];
#pragma unroll
        for (int c = 0; c < kBN; c += 2) {
          const float p0 = ex2(fmaf(s[c], sl2, -mu));
          const float p1 = ex2(fmaf(s[c + 1], sl2, -mu));
          l8[(c >> 1) & 7] += p0 + p1;
          pk[c >> 1] = pack_bf16x2(p0, p1);
        }
        l += ((l8[0] + l8[1]) + (l8[2] + l8[3])) + ((l8[4] + l8[5]) + (l8[6] + l8[7]));
        {
          uint32_t r[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = pk[e];
          tmem_st32(tS + sb * 128 + lane_off, r);
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = pk[32 + e];
          tmem_st32(tS + sb * 128 + 32 + lane_off, r);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(p_full + sb);
      }
      m_row[ps.sel] = m;
      l_row[ps.sel] = l;
    }

    // ------------------------------------------------------------ epilogue
    if (ok) ok = wwait(o_final, 0);
    if (ok) {
      tc_fence_after();
      const bool bif = p.kind == kBifocal;
      // per-accumulator weights: O = sum_X c_X * O_X, lse = (M + log2 W) ln 2
      float c0, c1 = 0.f, lse2;
      if (bif) {
        const float lg0 = l_row[0] > 0.f ? m_row[0] + __log2f(l_row[0]) : -INFINITY;
        const float lg1 = l_row[1] > 0.f ? m_row[1] + __log2f(l_row[1]) : -INFINITY;
        const float M = fmaxf(lg0, lg1);
        const float w0 = l_row[0] > 0.f ? ex2(lg0 - M) : 0.f;   // Eq. 7 weights W_X = exp(l_X - M)
        const float w1 = l_row[1] > 0.f ? ex2(lg1 - M) : 0.f;
        const float den = w0 + w1;
        c0 = l_row[0] > 0.f ? w0 / (l_row[0] * den) : 0.f;
        c1 = l_row[1] > 0.f ? w1 / (l_row[1] * den) : 0.f;
        lse2 = M + __log2f(den);
      } else {
        c0 = 1.0f / l_row[0];
        lse2 = m_row[0] + __log2f(l_row[0]);
      }
      float* orow = p.out + ((static_cast<size_t>(b) * p.S + (t < p.S ? t : 0)) * p.Hq + h) * D;
      uint32_t r0[32], r1[32];
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        tmem_ld32(tO + c * 32 + lane_off, r0);
        if (bif) tmem_ld32(tO + D + c * 32 + lane_off, r1);
        tmem_ld_wait();
        if (t < p.S) {
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            float4 o;
            o.x = __uint_as_float(r0[e + 0]) * c0;
            o.y = __uint_as_float(r0[e + 1]) * c0;
            o.z = __uint_as_float(r0[e + 2]) * c0;
            o.w = __uint_as_float(r0[e + 3]) * c0;
            if (bif) {
              o.x = fmaf(__uint_as_float(r1[e + 0]), c1, o.x);
              o.y = fmaf(__uint_as_float(r1[e + 1]), c1, o.y);
              o.z = fmaf(__uint_as_float(r1[e + 2]), c1, o.z);
              o.w = fmaf(__uint_as_float(r1[e + 3]), c1, o.w);
            }
            *reinterpret_cast<float4*>(orow + c * 32 + e) = o;
          }
        }
      }
      if (t < p.S) p.lse[(static_cast<size_t>(b) * p.Hq + h) * p.S + t] = lse2 * 0.69314718055994530942f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    // let in-flight TMA and MMA work drain before the CTA releases its memory
    const unsigned long long t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 20000000ull) __nanosleep(100000);
  }
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace ropeattn
