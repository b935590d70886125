// One decode step over an untouched RoPE key cache (Jet-Long §3.2), sm_100a.
//
// Split-KV: CTA (split, kv head, batch) owns a contiguous key range of one KV
// head; the grid is one wave (one CTA per SM). The range streams through a
// shared-memory ring by TMA, 64 keys per stage (no swizzle, no multicast).
// A lane group of 8 lanes holds D/8 dimensions of one key and of the query:
// 16 warps take one key per group per stage, or 8 warps two keys when the
// GQA group is too large for 128 registers a thread or D is 256. The last warp to
// release a slot issues the copy of the stage that reuses it; no thread polls.
//
// Scores: the query is rotated once to its position p(n-1) in fp32 and
// prescaled by softmax_scale * log2(e). For the bifocal map a remote key k
// ((n-1) - k > w0) is read through the correction of Eq. 6: with
// u(k) = k - f(k) = k - floor(k/G),
//   score = q_remote . R(-u(k)) k_cache,   q_remote = R(Delta q) q_local,
// and a local key through q_local . k_cache. R(-u(k)) is applied one of two
// ways (template parameter ROT):
//  * stage table (one key per group, any G): with d(r) = r - floor(r/G)
//    and phi = k0 mod G for the stage's first key k0,
//      u(k0 + r) = u(k0) + d(r) - e,  e = 1 if (r mod G) + phi >= G else 0,
//    so the group of row r keeps R(d(r)) q_remote, and the keys of a stage
//    share R(-u(k0)) (e = 0) or R(-(u(k0) - 1)) (e = 1; never when G divides
//    64, since every stage then starts at a multiple of G). Both (cos, sin)
//    tables are computed once per stage, NS stages ahead, by one warp (warp
//    st mod 16 while it works on stage st); the slot's barrier counts that
//    warp's arrival with the copy's. A group switches to q_local when its
//    keys become local.
//  * phasor recurrence (two keys per group): each lane carries exp(i u theta) for its
//    pairs and advances it by one complex multiply per stage, re-seeded
//    exactly every 16 stages; local keys use u(n-1), which turns
//    q_remote . R(Delta q) k_cache back into q_local . k_cache, so one query
//    view serves both windows.
// Every angle is an integer position times theta_i, taken from theta_i's
// fraction of a turn in 64-bit fixed point, so it is exact modulo a turn
// before the fp32 sincospi. Packed fp32x2 FMAs carry the rotation, the dot
// products and the accumulation.
//
// Each lane group keeps an online softmax per query head of the GQA group;
// the CTA merges its groups and warps, writes (O, m, l) for its split, and the
// last CTA of the (batch, kv head) to arrive merges all splits in split order.
#pragma once

#include "common.cuh"
#include "posmap.cuh"

namespace ropeattn {

constexpr int kDecKeys = 64;         // keys per stage
constexpr int kDecReseed = 16;       // stages between exact phasor re-seeds

// how remote keys are rotated
enum DecodeRot : int { kRotNone = 0, kRotTable = 1, kRotPhasor = 2 };

template <int D, int GRP>
struct DecodeShape {
  static constexpr int kKeysPerGroup = (GRP * D <= 256 && D <= 128) ? 1 : 2;
  static constexpr int kWarps = 16 / kKeysPerGroup;
  static constexpr int kThreads = kWarps * 32;
  static constexpr bool kMulInRegs = kKeysPerGroup == 2;   // phasor multipliers in registers
};

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

template <int D>
struct DecodeSmem {
  static constexpr int kStages = D == 256 ? 3 : (D == 128 ? 6 : 10);  // ring depth
  static constexpr int kRowBytes = D * 2;
  static constexpr int kStageBytes = 2 * kDecKeys * kRowBytes;  // K then V
  static constexpr int kRing = kStages * kStageBytes;
  static constexpr int kMul = kRing;                             // [2][D/2] float2 phasor stage multipliers
  static constexpr int kTab = kMul + D * 8;                      // [2 kStages][2][D/4] float4 stage tables
  static constexpr int kQloc = kTab + 4 * kStages * D * 4;       // [GRP][D/4] float4 local query view
  static constexpr int kBar = kQloc + 2048;                      // full[] mbarriers (GRP * D <= 512)
  static constexpr int kCnt = kBar + kStages * 8;                // release counters per slot
  static constexpr int kMisc = kCnt + kStages * 4;               // abort flag, last flag
  static constexpr int kTotal = kMisc + 16;
};

// Packed fp32x2 helpers (Blackwell FFMA2 / FMUL2).
__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 neg2(float2 a) { return make_float2(-a.x, -a.y); }

template <int D, int GRP, int ROT>
__global__ void __launch_bounds__(DecodeShape<D, GRP>::kThreads, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const DecodeParams p) {
  using L = DecodeSmem<D>;
  using SH = DecodeShape<D, GRP>;
  constexpr int NS = L::kStages;
  constexpr int NW = SH::kWarps;
  constexpr int NV = D / 64;              // 16-byte vectors per lane per row
  constexpr int NJ = 2 * NV;              // pair-pairs per lane (two rotation pairs each)
  constexpr int KPG = SH::kKeysPerGroup;  // keys per lane group per stage
  constexpr int RS = kDecKeys / KPG;      // row stride between a group's keys in a stage
  constexpr int NPP = D / 4;              // pair-pairs per row
  static_assert(GRP * D <= 512, "local query view table holds GRP * D <= 512 values");
  static_assert(ROT != kRotTable || KPG == 1, "stage tables need one key per group");

  extern __shared__ __align__(128) uint8_t smem[];
  float2* mul_tab = reinterpret_cast<float2*>(smem + L::kMul);   // [carry][pair] (cos, sin)
  float4* stab = reinterpret_cast<float4*>(smem + L::kTab);      // [slot][pair-pair] (c0, c1, s0, s1)
  float4* qloc = reinterpret_cast<float4*>(smem + L::kQloc);     // [gi][pair-pair] (q0 x2, q1 x2)
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBar);
  int* released = reinterpret_cast<int*>(smem + L::kCnt);
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
  const int G = p.m.G;
  const int stage_q = kDecKeys / G, stage_r = kDecKeys - stage_q * G;
  const int t = p.n - 1;                // query position index

  // Stage tables of stage st (table slot st mod 2 NS, variants e = 0, 1):
  // (cos, sin) of (u(k0) - e) theta for every pair, k0 the stage's first key;
  // variant 1 only when G does not divide 64. The entry of pair-pair pp
  // (pairs 2pp, 2pp+1) = (c0, c1, s0, s1) sits at
  // 16 (pp / 16) + 8 (pp % 2) + (pp % 16) / 2, so the 8 lanes of a group read
  // 128 consecutive bytes. One warp writes them, then arrives on the stage's
  // ring barrier.
  const bool two_tabs = (kDecKeys % G) != 0;
  auto tab_pos = [](int pp) { return 16 * (pp >> 4) + 8 * (pp & 1) + ((pp & 15) >> 1); };
  auto fill_table = [&](int st) {
    const int k0 = kb + st * kDecKeys;
    const int u0 = k0 - k0 / G;
    for (int e = 0; e < (two_tabs ? 2 : 1); ++e) {
      float4* tab = stab + ((st % (2 * NS)) * 2 + e) * NPP;
      for (int pp = lane; pp < NPP; pp += 32) {
        const float2 x = turn_cs(u0 - e, p.turns[2 * pp]);
        const float2 y = turn_cs(u0 - e, p.turns[2 * pp + 1]);
        tab[tab_pos(pp)] = make_float4(x.x, y.x, x.y, y.y);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(full + st % NS);
  };
  auto issue = [&](int st) {  // copy stage st (K rows then V rows) into its slot
    const int slot = st % NS;
    uint8_t* dst = smem + slot * L::kStageBytes;
    mbar_arrive_expect_tx(full + slot, L::kStageBytes);
    tma_load_4d(dst, &tmK, full + slot, 0, hkv, kb + st * kDecKeys, b);
    tma_load_4d(dst + kDecKeys * L::kRowBytes, &tmV, full + slot, 0, hkv, kb + st * kDecKeys, b);
  };
  if (tid == 0) {
    // the copy's arrival, plus the stage table's
    const uint32_t arrivals = ROT == kRotTable ? 2 : 1;
    for (int i = 0; i < NS; ++i) {
      mbar_init(full + i, arrivals);
      released[i] = 0;
    }
    *abort_flag = 0;
    *last_flag = 0;
    mbar_fence_init();
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    for (int st = 0; st < NS && st < nstage; ++st) issue(st);
  }
  if constexpr (ROT == kRotPhasor) {
    // per pair: (cos, sin) of the stage advance of u without and with a
    // group-boundary carry: 64 - 64/G and 63 - 64/G positions
    for (int i = tid; i < D / 2; i += SH::kThreads) {
      const int du = kDecKeys - stage_q;
      mul_tab[i] = turn_cs(du, p.turns[i]);
      mul_tab[D / 2 + i] = turn_cs(du - 1, p.turns[i]);
    }
  }
  // local query view R(p(t)) q prescaled by softmax scale * log2(e): entry
  // (q0 of pairs 2pp, 2pp+1; q1 of pairs 2pp, 2pp+1) per pair-pair
  if (tid >= 32 && tid < 32 + GRP * NPP) {
    const int i = tid - 32, gi = i / NPP, pp = i % NPP;
    const int hq = hkv * GRP + gi;
    const uint2 xq = __ldg(reinterpret_cast<const uint2*>(p.q + (static_cast<size_t>(b) * p.Hq + hq) * D) + pp);
    const int pq = pos_primary(p.m, t);
    const uint32_t xw[2] = {xq.x, xq.y};
    float r0[2], r1[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float a0 = bf16lo(xw[e]), a1 = bf16hi(xw[e]);
      if (p.m.kind != kNope) {
        const float2 cs = turn_cs(pq, p.turns[2 * pp + e]);
        rot_pair(bf16lo(xw[e]), bf16hi(xw[e]), cs.x, cs.y, a0, a1);
      }
      r0[e] = a0 * p.scale_log2;
      r1[e] = a1 * p.scale_log2;
    }
    qloc[gi * NPP + pp] = make_float4(r0[0], r0[1], r1[0], r1[1]);
  }
  __syncthreads();
  if constexpr (ROT == kRotTable) {
    if (warp < NS && warp < nstage) fill_table(warp);
  }

  const int j4 = lane >> 3;             // lane group within the warp
  const int l8 = lane & 7;              // lane within the group
  const int ks = warp * 4 + j4;         // key stream: rows ks + RS * kk of every stage
  const unsigned gmask = 0xFFu << (8 * j4);
  const int u_t = t - t / G;            // u of the query: local keys are read at u(t)
  // Lane pair-pair j holds rotation pairs c = 0, 1 at word 2(j%2)+c of the
  // 16-byte vector j/2: global pair 32 (j/2) + 4 l8 + 2 (j%2) + c, i.e.
  // global pair-pair 16 (j/2) + 2 l8 + (j%2).
  auto gpair = [&](int j, int c) { return 32 * (j >> 1) + 4 * l8 + 2 * (j & 1) + c; };
  auto gpp = [&](int j) { return 16 * (j >> 1) + 2 * l8 + (j & 1); };
  const float2 kNeg = f2(-1.f, -1.f);

  float2 Q0[GRP][NJ], Q1[GRP][NJ];
  auto load_local = [&]() {
#pragma unroll
    for (int gi = 0; gi < GRP; ++gi)
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        const float4 x = qloc[gi * NPP + gpp(j)];
        Q0[gi][j] = f2(x.x, x.y);
        Q1[gi][j] = f2(x.z, x.w);
      }
  };
  // rotate the query view by +shift positions
  auto rotate_query = [&](int shift) {
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      const float2 x = turn_cs(shift, p.turns[gpair(j, 0)]);
      const float2 y = turn_cs(shift, p.turns[gpair(j, 1)]);
      const float2 C = f2(x.x, y.x), Sn = f2(x.y, y.y);
#pragma unroll
      for (int gi = 0; gi < GRP; ++gi) {
        // (a0 c - a1 s, a0 s + a1 c)
        const float2 y0 = fma2(mul2(Q1[gi][j], kNeg), Sn, mul2(Q0[gi][j], C));
        const float2 y1 = fma2(Q0[gi][j], Sn, mul2(Q1[gi][j], C));
        Q0[gi][j] = y0;
        Q1[gi][j] = y1;
      }
    }
  };
  load_local();
  const int dq = pos_remote(p.m, t) - t;   // Delta q (Eq. 5)
  bool q_remote = false;                   // stage-table view: query currently R(d(ks)) q_remote
  if constexpr (ROT == kRotPhasor) rotate_query(dq);
  if constexpr (ROT == kRotTable) {
    q_remote = kb + ks < p.k_local;
    if (q_remote) rotate_query(dq + (ks - ks / G));
  }

  // phasor recurrence state: exp(i u theta) of the stream's keys (u = u(k)
  // for remote keys, u(t) for local ones) and the no-carry stage multiplier
  int a0[KPG], r0[KPG];
  float2 PC[KPG][NJ], PS[KPG][NJ];
  float2 MC[NJ], MS[NJ], MSN[NJ];
  auto seed = [&](int kk, int u) {
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      const float2 x = turn_cs(u, p.turns[gpair(j, 0)]);
      const float2 y = turn_cs(u, p.turns[gpair(j, 1)]);
      PC[kk][j] = f2(x.x, y.x);
      PS[kk][j] = f2(x.y, y.y);
    }
  };
  if constexpr (ROT == kRotPhasor) {
#pragma unroll
    for (int kk = 0; kk < KPG; ++kk) {
      const int k = kb + ks + RS * kk;
      a0[kk] = k / G;
      r0[kk] = k - a0[kk] * G;
      seed(kk, k < p.k_local ? k - a0[kk] : u_t);
    }
    if constexpr (SH::kMulInRegs) {
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        const float2 x = mul_tab[gpair(j, 0)], y = mul_tab[gpair(j, 1)];
        MC[j] = f2(x.x, y.x);
        MS[j] = f2(x.y, y.y);
        MSN[j] = f2(-x.y, -y.y);
      }
    }
  }

  float m_run[GRP], l_run[GRP];
  float2 A0[GRP][NJ], A1[GRP][NJ];
#pragma unroll
  for (int gi = 0; gi < GRP; ++gi) {
    m_run[gi] = -INFINITY;
    l_run[gi] = 0.f;
#pragma unroll
    for (int j = 0; j < NJ; ++j) A0[gi][j] = A1[gi][j] = f2(0.f, 0.f);
  }

  bool ok = true;
  int slot = 0, tslot = 0;
  uint32_t phase = 0;
  int phi = kb % G;                       // first key of the current stage, mod G
  const int adv = kDecKeys % G, ks_mod = ks % G;
  // one stage of 64 keys; all_remote: every key of the stage is a remote key
  // (the stage-table path then rotates unconditionally)
  auto stage_step = [&](const int st, const bool all_remote) -> bool {
    if (!__all_sync(0xffffffffu, mbar_wait(full + slot, phase, abort_flag))) return false;
    const int k0 = kb + st * kDecKeys + ks;
    const uint8_t* rows = smem + slot * L::kStageBytes + ks * L::kRowBytes;
    uint4 kr[KPG][NV], vr[KPG][NV];
    float4 tb[NJ];
    const bool rem_t = ROT == kRotTable && (all_remote || k0 < p.k_local);
#pragma unroll
    for (int kk = 0; kk < KPG; ++kk)
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        kr[kk][v] = *reinterpret_cast<const uint4*>(rows + RS * kk * L::kRowBytes + v * 128 + l8 * 16);
        vr[kk][v] = *reinterpret_cast<const uint4*>(rows + (kDecKeys + RS * kk) * L::kRowBytes + v * 128 + l8 * 16);
      }
    if constexpr (ROT == kRotTable) {
      if (rem_t) {
        const float4* tt = stab + (tslot * 2 + (phi + ks_mod >= G ? 1 : 0)) * NPP;
#pragma unroll
        for (int j = 0; j < NJ; ++j) tb[j] = tt[16 * (j >> 1) + 8 * (j & 1) + l8];
      }
    }
    __syncwarp();
    if (lane == 0) {
      // the last warp to release the slot refills it with stage st + NS: the
      // block fences and the counter order every warp's (generic) reads of the
      // slot before the last release, and the proxy fence orders them before
      // the copy engine's (async proxy) writes into the slot
      __threadfence_block();
      if (atomicAdd(released + slot, 1) == NW - 1) {
        __threadfence_block();
        released[slot] = 0;
        fence_proxy_async_smem();
        if (st + NS < nstage) issue(st + NS);
      }
    }

    float sc[KPG][GRP];
#pragma unroll
    for (int kk = 0; kk < KPG; ++kk) {
      float2 X0[NJ], X1[NJ];
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        const uint4 w = kr[kk][j >> 1];
        const uint32_t wa = (j & 1) ? w.z : w.x, wb = (j & 1) ? w.w : w.y;
        X0[j] = f2(bf16lo(wa), bf16lo(wb));
        X1[j] = f2(bf16hi(wa), bf16hi(wb));
      }
      if constexpr (ROT == kRotPhasor) {
        // R(-u theta) k_cache: (x0 c + x1 s, x1 c - x0 s)
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
          const float2 y0 = fma2(X1[j], PS[kk][j], mul2(X0[j], PC[kk][j]));
          const float2 y1 = fma2(mul2(X0[j], kNeg), PS[kk][j], mul2(X1[j], PC[kk][j]));
          X0[j] = y0;
          X1[j] = y1;
        }
      }
      if constexpr (ROT == kRotTable) {
        if (rem_t) {
          // R(-u(k0) theta) k_cache with the stage's shared table
#pragma unroll
          for (int j = 0; j < NJ; ++j) {
            const float2 C = f2(tb[j].x, tb[j].y), Sn = f2(tb[j].z, tb[j].w);
            const float2 y0 = fma2(X1[j], Sn, mul2(X0[j], C));
            const float2 y1 = fma2(neg2(X0[j]), Sn, mul2(X1[j], C));
            X0[j] = y0;
            X1[j] = y1;
          }
        } else if (!all_remote && q_remote) {
          // this stream's keys became local: exact-position query view
          load_local();
          q_remote = false;
        }
      }
#pragma unroll
      for (int gi = 0; gi < GRP; ++gi) {
        float2 acc0 = mul2(Q0[gi][0], X0[0]);
        float2 acc1 = mul2(Q1[gi][0], X1[0]);
#pragma unroll
        for (int j = 1; j < NJ; ++j) {
          acc0 = fma2(Q0[gi][j], X0[j], acc0);
          acc1 = fma2(Q1[gi][j], X1[j], acc1);
        }
        const float2 a = __fadd2_rn(acc0, acc1);
        sc[kk][gi] = a.x + a.y;
      }
    }
#pragma unroll
    for (int off = 1; off <= 4; off <<= 1)
#pragma unroll
      for (int kk = 0; kk < KPG; ++kk)
#pragma unroll
        for (int gi = 0; gi < GRP; ++gi) sc[kk][gi] += __shfl_xor_sync(gmask, sc[kk][gi], off);
    bool vk[KPG];
#pragma unroll
    for (int kk = 0; kk < KPG; ++kk) vk[kk] = k0 + RS * kk < ke;
#pragma unroll
    for (int gi = 0; gi < GRP; ++gi) {
      float mx = -INFINITY;
#pragma unroll
      for (int kk = 0; kk < KPG; ++kk) {
        sc[kk][gi] = vk[kk] ? sc[kk][gi] : -INFINITY;
        mx = fmaxf(mx, sc[kk][gi]);
      }
      if (mx > m_run[gi]) {
        const float corr = ex2(m_run[gi] - mx);
        l_run[gi] *= corr;
        const float2 c2 = f2(corr, corr);
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
          A0[gi][j] = mul2(A0[gi][j], c2);
          A1[gi][j] = mul2(A1[gi][j], c2);
        }
        m_run[gi] = mx;
      }
#pragma unroll
      for (int kk = 0; kk < KPG; ++kk) {
        sc[kk][gi] = vk[kk] ? ex2(sc[kk][gi] - m_run[gi]) : 0.f;
        l_run[gi] += sc[kk][gi];
      }
    }
#pragma unroll
    for (int kk = 0; kk < KPG; ++kk) {
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        const uint4 w = vr[kk][j >> 1];
        const uint32_t wa = (j & 1) ? w.z : w.x, wb = (j & 1) ? w.w : w.y;
        const float2 V0 = f2(bf16lo(wa), bf16lo(wb));
        const float2 V1 = f2(bf16hi(wa), bf16hi(wb));
#pragma unroll
        for (int gi = 0; gi < GRP; ++gi) {
          const float2 p2 = f2(sc[kk][gi], sc[kk][gi]);
          A0[gi][j] = fma2(p2, V0, A0[gi][j]);
          A1[gi][j] = fma2(p2, V1, A1[gi][j]);
        }
      }
    }

    // advance the phasors to the keys of the next stage
    if constexpr (ROT == kRotPhasor) {
      const bool reseed_now = ((st + 1) % kDecReseed) == 0;
#pragma unroll
      for (int kk = 0; kk < KPG; ++kk) {
        const int k = k0 + RS * kk;
        const int kn = k + kDecKeys;
        r0[kk] += stage_r;
        const bool carry = r0[kk] >= G;
        if (carry) r0[kk] -= G;
        a0[kk] += stage_q + (carry ? 1 : 0);
        if (kn >= ke || k >= p.k_local) continue;        // no next key, or already at u(t)
        if (kn >= p.k_local) {
          seed(kk, u_t);                                  // entering the local window
        } else if (reseed_now) {
          seed(kk, kn - a0[kk]);
        } else if (!carry && SH::kMulInRegs) {
#pragma unroll
          for (int j = 0; j < NJ; ++j) {
            const float2 c = fma2(PC[kk][j], MC[j], mul2(PS[kk][j], MSN[j]));
            const float2 sn = fma2(PC[kk][j], MS[j], mul2(PS[kk][j], MC[j]));
            PC[kk][j] = c;
            PS[kk][j] = sn;
          }
        } else {
#pragma unroll
          for (int j = 0; j < NJ; ++j) {
            const int base = carry ? D / 2 : 0;
            const float2 x = mul_tab[base + gpair(j, 0)], y = mul_tab[base + gpair(j, 1)];
            const float2 mc = f2(x.x, y.x), ms = f2(x.y, y.y);
            const float2 c = fma2(PC[kk][j], mc, mul2(PS[kk][j], mul2(ms, kNeg)));
            const float2 sn = fma2(PC[kk][j], ms, mul2(PS[kk][j], mc));
            PC[kk][j] = c;
            PS[kk][j] = sn;
          }
        }
      }
    }
    // the table of the stage that reuses the slot, by one warp in turn
    if constexpr (ROT == kRotTable) {
      if (warp == st % NW && st + NS < nstage) fill_table(st + NS);
    }
    if (++tslot == 2 * NS) tslot = 0;
    phi += adv;
    if (phi >= G) phi -= G;
    if (++slot == NS) {
      slot = 0;
      phase ^= 1u;
    }
    return true;
  };
  // stages whose 64 keys all lie before the local window first, without the
  // per-key remote/local test, then the rest
  int st = 0;
  if constexpr (ROT == kRotTable) {
    const int st_rem = min(nstage, p.k_local - kb >= kDecKeys ? (p.k_local - kb) / kDecKeys : 0);
    for (; st < st_rem && ok; ++st) ok = stage_step(st, true);
  }
  for (; st < nstage && ok; ++st) ok = stage_step(st, false);

  // --------------------------------------------- merge lane groups of a warp
#pragma unroll
  for (int gi = 0; gi < GRP; ++gi) {
#pragma unroll
    for (int off = 8; off <= 16; off <<= 1) {
      const float mo = __shfl_xor_sync(0xffffffffu, m_run[gi], off);
      const float lo = __shfl_xor_sync(0xffffffffu, l_run[gi], off);
      const float M = fmaxf(m_run[gi], mo);
      const float fa = (l_run[gi] > 0.f) ? ex2(m_run[gi] - M) : 0.f;
      const float fb = (lo > 0.f) ? ex2(mo - M) : 0.f;
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        float2 o0, o1;
        o0.x = __shfl_xor_sync(0xffffffffu, A0[gi][j].x, off);
        o0.y = __shfl_xor_sync(0xffffffffu, A0[gi][j].y, off);
        o1.x = __shfl_xor_sync(0xffffffffu, A1[gi][j].x, off);
        o1.y = __shfl_xor_sync(0xffffffffu, A1[gi][j].y, off);
        A0[gi][j] = fma2(A0[gi][j], f2(fa, fa), mul2(o0, f2(fb, fb)));
        A1[gi][j] = fma2(A1[gi][j], f2(fa, fa), mul2(o1, f2(fb, fb)));
      }
      l_run[gi] = l_run[gi] * fa + lo * fb;
      m_run[gi] = M;
    }
  }
  // -------------------------------------------------- merge warps via smem
  // (the ring is free: every issued stage was waited for above; after an
  // abort the buffers may still be written by a late copy, and the results
  // are void anyway)
  __syncthreads();
  float* red_o = reinterpret_cast<float*>(smem);                       // [NW][GRP][D]
  float2* red_ml = reinterpret_cast<float2*>(smem + NW * GRP * D * 4);  // [NW][GRP]
  if (j4 == 0) {
#pragma unroll
    for (int gi = 0; gi < GRP; ++gi) {
      float* dst = red_o + (warp * GRP + gi) * D;
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        const int g0 = gpair(j, 0), g1 = gpair(j, 1);
        dst[2 * g0] = A0[gi][j].x;
        dst[2 * g0 + 1] = A1[gi][j].x;
        dst[2 * g1] = A0[gi][j].y;
        dst[2 * g1 + 1] = A1[gi][j].y;
      }
      if (l8 == 0) red_ml[warp * GRP + gi] = make_float2(m_run[gi], l_run[gi]);
    }
  }
  __syncthreads();
  for (int idx = tid; idx < GRP * D; idx += SH::kThreads) {
    const int gi = idx / D, d = idx % D;
    float M = -INFINITY;
    for (int w = 0; w < NW; ++w) {
      const float2 ml = red_ml[w * GRP + gi];
      if (ml.y > 0.f) M = fmaxf(M, ml.x);
    }
    float o = 0.f, l = 0.f;
    for (int w = 0; w < NW; ++w) {
      const float2 ml = red_ml[w * GRP + gi];
      if (ml.y > 0.f) {
        const float f = ex2(ml.x - M);
        o = fmaf(red_o[(w * GRP + gi) * D + d], f, o);
        l = fmaf(ml.y, f, l);
      }
    }
    const int hq = hkv * GRP + gi;
    const size_t pslot = (static_cast<size_t>(b) * p.Hq + hq) * p.nsplit + split;
    p.part_o[pslot * D + d] = o;
    if (d == 0) p.part_ml[pslot] = make_float2(M, l);
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const int prev = atomicAdd(p.counters + b * p.Hkv + hkv, 1);
    *last_flag = (prev == p.nsplit - 1) ? 1 : 0;
  }
  __syncthreads();
  if (*last_flag) {
    // last CTA of this (batch, kv head): merge every split, in split order
    __threadfence();
    for (int idx = tid; idx < GRP * D; idx += SH::kThreads) {
      const int gi = idx / D, d = idx % D;
      const int hq = hkv * GRP + gi;
      const size_t base = (static_cast<size_t>(b) * p.Hq + hq) * p.nsplit;
      float M = -INFINITY;
      for (int sp = 0; sp < p.nsplit; ++sp) {
        const float2 ml = __ldcg(p.part_ml + base + sp);
        if (ml.y > 0.f) M = fmaxf(M, ml.x);
      }
      float o = 0.f, l = 0.f;
      for (int sp = 0; sp < p.nsplit; ++sp) {
        const float2 ml = __ldcg(p.part_ml + base + sp);
        if (ml.y > 0.f) {
          const float f = ex2(ml.x - M);
          o = fmaf(__ldcg(p.part_o + (base + sp) * D + d), f, o);
          l = fmaf(ml.y, f, l);
        }
      }
      p.out[(static_cast<size_t>(b) * p.Hq + hq) * D + d] = o / l;
      if (d == 0) p.lse[static_cast<size_t>(b) * p.Hq + hq] = (M + __log2f(l)) * 0.69314718055994530942f;
    }
    if (tid == 0) p.counters[b * p.Hkv + hkv] = 0;
  }
  if (*abort_flag) {
    const unsigned long long t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 20000000ull) __nanosleep(100000);
  }
  (void)ok;
}

}  // namespace ropeattn
