// Causal prefill attention with RoPE at remapped positions, sm_100a.
//
// One CTA computes two 128-row query tiles (256 consecutive rows) of one
// (batch, query head) against the 128-key tiles of its passes (D = 64, 128;
// at D = 256 one query tile against 64-key tiles, see PrefillShape):
//   warps 0-3, 4-7  softmax warpgroups, one per query tile (one TMEM lane =
//              one query row per thread): rotate the staged query tile in
//              shared memory, then per key tile copy S from TMEM into
//              registers (and release S at once), mask, online softmax in the
//              exp2 domain, write P (bf16) to the tile's own TMEM columns,
//              and at the end normalise, merge and store O and the LSE.
//   warp 8     TMA producer: the query tiles, then K and V tiles through one
//              ring of NSLOT tile slots (128-byte swizzle, no multicast).
//   warp 9     QK issuer (one thread), per key tile j: S = Q0 K_j^T, then
//              S = Q1 K_j^T. Both tiles share one S buffer: a QK only waits
//              until the previous S has been copied into registers by its
//              softmax, so the QKs of the next key tile overlap the
//              exponentials of this one.
//   warps 10, 11  PV issuers (one thread each), per key tile j:
//              O_a += P_a(j) V_j for tile a = warp - 10, once P_a is stored.
//              Separate issuers split the barrier waits and commits (each
//              costs the issuing thread about a hundred cycles, and the issue
//              queue is about one MMA deep), so one keeps the tensor pipe fed
//              while another waits. A softmax computes its row of P into
//              registers, then waits for its tile's previous PV (one barrier
//              per tile, committed after each PV) before rescaling O or
//              overwriting P, so its exponentials overlap that PV.
//   Registers: warps 8-11 (the third warpgroup) hand theirs to the softmax
//              warpgroups with setmaxnreg: 216 per softmax thread, 72 per
//              thread of warps 8-11; 384 x 168 at launch = 256 x 216 + 128 x 72.
// TMEM (512 columns): S [0,128), P0 [128,192), P1 [192,256) (bf16 pairs),
// O0 [256,256+D), O1 [256+D, 256+2D). At D = 256 the single tile's S, P and
// O take [0,64), [128,160) and [256,512); the warp roles shift down by the
// missing softmax warpgroup (TMA warp 4, QK warp 5, PV warp 6), and every
// thread keeps its launch registers (seven warps are not whole warpgroups,
// and 224 threads x 255 registers fit the register file).
//
// A pass is a sweep over key tiles with one query rotation, one key tensor
// and one distance band hi_off <= t - s <= lo_off:
//   standard / EndPrompt / NoPE: one pass, band [0, inf) (causal);
//   Periodic RoPE: one pass, band [0, W-1] (the window {t-W+1..t}, §3.2);
//   Jet-Long bifocal: a remote pass, band [w0+1, inf), with remote query
//   and keys, then a local pass, band [0, w0], with exact positions (Eq. 1).
// The two bifocal passes are the remote-only term W_B O_B - W_C O_C and the
// call-A term of the inclusion-exclusion merge (Jet-Long §3.3 Eq. 7),
// obtained by masking instead of subtraction. The remote partial (normalised)
// is parked in the output rows, the query tiles are reloaded and rotated to
// exact positions, and the local pass's epilogue merges the two by their
// log-sum-exp weights in fp32. A forced single pass (one band and map, own
// output) serves the literal three-call route; a query-row offset and a key
// count apart from the query rows serve chunked prefill from a cache.
// CTAs are ordered kv-head-major, so the resident CTAs stream the keys and
// values of about one kv head and keep them in L2.
#pragma once

#include "common.cuh"
#include "posmap.cuh"

namespace ropeattn {

constexpr int kBM = 128;               // rows per query tile (TMEM lanes)
constexpr int kSoftmaxRegs = 216;      // per thread of warps 0-7 after setmaxnreg (two tiles)
constexpr int kProducerRegs = 72;      // per thread of warps 8-11 after setmaxnreg (two tiles)
constexpr int kInf = 0x3fffffff;

// Tile schedule per head dimension. D <= 128: two query tiles per CTA, 128
// keys per tile. D = 256: one query tile per CTA (its O accumulator takes 256
// TMEM columns) and 64 keys per tile (a 64 KiB query tile and four 32 KiB
// K/V slots fit shared memory).
template <int D>
struct PrefillShape {
  static constexpr int kQT = D == 256 ? 1 : 2;          // query tiles per CTA
  static constexpr int kBN = D == 256 ? 64 : 128;       // keys per tile
  static constexpr int kBlockRows = kBM * kQT;          // query rows per CTA
  static constexpr int kWarpTMA = 4 * kQT;              // warp roles after the softmax warps
  static constexpr int kWarpQK = kWarpTMA + 1;
  static constexpr int kWarpPV = kWarpTMA + 2;          // kQT PV issuers
  static constexpr int kThreads = 32 * (kWarpPV + kQT);
};

struct PrefillParams {
  float* out;          // [B, S, Hq, D]
  float* lse;          // [B, Hq, S]
  const float2* tab0;  // [S][D/2] query (cos, sin) at map-0 positions (null for NoPE)
  const float2* tab1;  // [S][D/2] at remote positions (bifocal)
  int B, S, Hq, Hkv;   // S: query rows
  int Sk;              // keys (rows of K and V); S for a whole prefill
  int q_off;           // absolute position index of query row 0 (0 for a whole prefill)
  int nqb;             // query blocks (PrefillShape::kBlockRows rows) per (b, h)
  int kind;
  int window;          // Periodic RoPE
  int w0;              // Jet-Long
  float scale_log2;    // softmax scale * log2(e)
  // one forced pass (the separate calls of the literal three-call bifocal
  // prefill): band hi <= t - s <= lo with query/key map sel; 0 = off
  int forced, forced_lo, forced_hi, forced_sel;
};

struct PassDesc {
  int j_lo, j_hi;      // key tiles [j_lo, j_hi]
  int lo_off, hi_off;  // allowed band: hi_off <= t - s <= lo_off
  int sel;             // 0: main or local map, 1: remote map
};

__device__ __forceinline__ int make_passes(const PrefillParams& p, int q0, int block_rows, int bn, PassDesc* ps) {
  int bands[2][3];  // lo_off, hi_off, sel
  int nb = 0;
  if (p.forced) {
    bands[0][0] = p.forced_lo; bands[0][1] = p.forced_hi; bands[0][2] = p.forced_sel;
    nb = 1;
  } else if (p.kind == kBifocal) {
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
  // absolute positions of the block's first and last query rows
  const int t_first = p.q_off + q0;
  const int t_last = p.q_off + min(p.S - 1, q0 + block_rows - 1);
  int n = 0;
  for (int i = 0; i < nb; ++i) {
    const int lo_off = bands[i][0], hi_off = bands[i][1];
    const int s_min = lo_off >= kInf ? 0 : max(0, t_first - lo_off);
    const int s_max = min(p.Sk - 1, t_last - hi_off);
    if (s_max < s_min) continue;
    ps[n].j_lo = s_min / bn;
    ps[n].j_hi = s_max / bn;
    ps[n].lo_off = lo_off;
    ps[n].hi_off = hi_off;
    ps[n].sel = bands[i][2];
    ++n;
  }
  return n;
}

template <int D, int NSLOT>
struct PrefillSmem {
  static constexpr int kQBytes = kBM * D * 2;                       // one query tile
  static constexpr int kTileBytes = PrefillShape<D>::kBN * D * 2;   // one K or V tile
  static constexpr int kQ = 0;
  // at D = 256 the rotated query tile lives in TMEM and arrives through two
  // ring slots, so the ring takes the whole space (six 32 KiB slots)
  static constexpr int kRing = kQ + (D == 256 ? 0 : PrefillShape<D>::kQT * kQBytes);
  static constexpr int kBar = kRing + NSLOT * kTileBytes;
  // barriers: q_full, q_ready[2], q_free, ring_full[NSLOT], ring_empty[NSLOT],
  // s_full[2], s_free, p_full[2], o_done[2], o_free[2]
  static constexpr int kNumBars = 13 + 2 * NSLOT;
  static constexpr int kMisc = kBar + kNumBars * 8;  // tmem base (u32), abort flag (int)
  static constexpr int kTotal = kMisc + 16;
  static constexpr int kAlloc = kTotal + 1024;       // slack to align the base to 1024
};

template <int D, int NSLOT>
__global__ void __launch_bounds__(PrefillShape<D>::kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK0,
                   const __grid_constant__ CUtensorMap tmK1, const __grid_constant__ CUtensorMap tmV,
                   const PrefillParams p) {
  using L = PrefillSmem<D, NSLOT>;
  using SH = PrefillShape<D>;
  constexpr int kQT = SH::kQT;
  constexpr int kBN = SH::kBN;
  constexpr int kBlockRows = SH::kBlockRows;
  static_assert(NSLOT % 2 == 0, "K and V tiles alternate over an even number of ring slots");
  constexpr int kCB = D / 64;              // 64-column (128-byte) swizzle blocks per row
  constexpr int kBlockBytes = kBM * 128;   // one swizzle block of a query tile
  constexpr int kKVBlockBytes = kBN * 128; // one swizzle block of a K or V tile
  constexpr uint32_t kIdescQK = idesc_bf16_f32(kBM, kBN, false);
  constexpr uint32_t kIdescPV = idesc_bf16_f32(kBM, D, true);
  constexpr uint32_t kTmemCols = 512;
  // D = 256: the rotated query tile is the A operand of QK^T from TMEM
  // (128 lanes x 128 columns of bf16 pairs), staged through two ring slots
  constexpr bool kQTmem = D == 256;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + L::kQ;
  uint8_t* sRing = smem + L::kRing;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* q_full = bars + 0;
  uint64_t* q_ready = bars + 1;            // [2]
  uint64_t* q_free = bars + 3;
  uint64_t* ring_full = bars + 4;          // [NSLOT]
  uint64_t* ring_empty = ring_full + NSLOT;
  uint64_t* s_full = ring_empty + NSLOT;   // [2] S holds Q_a K^T
  uint64_t* s_free = s_full + 2;           // S copied out by a softmax warpgroup
  uint64_t* p_full = s_free + 1;           // [2]
  uint64_t* o_done = p_full + 2;           // [2] PV of tile a completed
  uint64_t* o_free = o_done + 2;           // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  // work item, kv-head-major: all query blocks (longest first) and query
  // heads of one (batch, kv head) before the next, so the CTAs resident at
  // any time stream the keys and values of few kv heads and keep them in L2
  const int grp = p.Hq / p.Hkv;
  const int per_kv = p.nqb * grp;
  const int bh = static_cast<int>(blockIdx.x) / per_kv;
  const int r2 = static_cast<int>(blockIdx.x) % per_kv;
  const int b = bh / p.Hkv;
  const int hk = bh % p.Hkv;
  const int qb = p.nqb - 1 - r2 / grp;
  const int h = hk * grp + r2 % grp;
  const int q0 = qb * kBlockRows;

  PassDesc passes[2];
  const int npass = make_passes(p, q0, kBlockRows, kBN, passes);

  if (tid == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_ready + 0, kBM);
    mbar_init(q_ready + 1, kBM);
    mbar_init(q_free, 1);
    // K tiles sit at even ring positions (released by the QK issuer), V tiles
    // at odd ones (released by every PV issuer); NSLOT is even
    for (int i = 0; i < NSLOT; ++i) {
      mbar_init(ring_full + i, 1);
      mbar_init(ring_empty + i, (i & 1) ? kQT : 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(s_full + a, 1);
      mbar_init(p_full + a, kBM);
      mbar_init(o_done + a, 1);
      mbar_init(o_free + a, kBM);
    }
    mbar_init(s_free, kBM);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == SH::kWarpTMA && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK0);
    tma_prefetch_desc(&tmK1);
    tma_prefetch_desc(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem;            // S, shared by the two tiles
  // P_a at 128 + 64 a; at D = 256: S [0,64), Q [64,192), P [192,224)
  const uint32_t tP = tmem + (kQTmem ? 192 : 128);
  const uint32_t tQ = tmem + 64;       // D = 256 only
  const uint32_t tO = tmem + 256;      // O_a at 256 + a D

  if (warp == SH::kWarpTMA) {
    // ------------------------------------------------------------------ TMA
    if constexpr (kQT == 2) reg_dealloc<kProducerRegs>();
    if (lane == 0) {
      int pos = 0;
      bool ok = true;
      for (int pi = 0; pi < npass && ok; ++pi) {
        if constexpr (kQTmem) {
          // the query tile through the next two ring positions (even, so
          // the two slots are adjacent): its 64-column blocks 0-1, then 2-3
          for (int hq = 0; hq < 2 && ok; ++hq, ++pos) {
            const int slot = pos % NSLOT;
            if (!mbar_wait(ring_empty + slot, ((pos / NSLOT) & 1) ^ 1, abort_flag)) { ok = false; break; }
            mbar_arrive_expect_tx(ring_full + slot, L::kTileBytes);
            for (int cb = 2 * hq; cb < 2 * hq + 2; ++cb)
              tma_load_4d(sRing + slot * L::kTileBytes + (cb - 2 * hq) * kBlockBytes, &tmQ, ring_full + slot,
                          cb * 64, h, q0, b);
          }
          if (!ok) break;
        } else {
          // the query tiles of the previous pass must no longer be read
          if (pi > 0 && !mbar_wait(q_free, (pi - 1) & 1, abort_flag)) break;
          mbar_arrive_expect_tx(q_full, kQT * L::kQBytes);
          for (int a = 0; a < kQT; ++a)
            for (int cb = 0; cb < kCB; ++cb)
              tma_load_4d(sQ + a * L::kQBytes + cb * kBlockBytes, &tmQ, q_full, cb * 64, h, q0 + a * kBM, b);
        }
        const CUtensorMap* tk = passes[pi].sel ? &tmK1 : &tmK0;
        for (int j = passes[pi].j_lo; j <= passes[pi].j_hi && ok; ++j) {
          for (int kv = 0; kv < 2; ++kv, ++pos) {
            const int slot = pos % NSLOT;
            if (!mbar_wait(ring_empty + slot, ((pos / NSLOT) & 1) ^ 1, abort_flag)) { ok = false; break; }
            mbar_arrive_expect_tx(ring_full + slot, L::kTileBytes);
            uint8_t* dst = sRing + slot * L::kTileBytes;
            for (int cb = 0; cb < kCB; ++cb)
              tma_load_4d(dst + cb * kKVBlockBytes, kv ? &tmV : tk, ring_full + slot, cb * 64, hk, j * kBN, b);
          }
        }
      }
    }
  } else if (warp == SH::kWarpQK) {
    // ---------------------------------------------------------- MMA: QK^T
    if constexpr (kQT == 2) reg_dealloc<kProducerRegs>();
    if (lane == 0) {
      int pos = 0, nqk = 0;
      bool ok = true;
      for (int pi = 0; pi < npass && ok; ++pi) {
        if (!mbar_wait(q_ready + 0, pi & 1, abort_flag) ||
            (kQT == 2 && !mbar_wait(q_ready + 1, pi & 1, abort_flag)))
          break;
        if constexpr (kQTmem) {
          // every softmax thread has read the query tile's two ring slots
          // (and stored it in TMEM): hand the slots back to the producer
          mbar_arrive(ring_empty + pos % NSLOT);
          mbar_arrive(ring_empty + (pos + 1) % NSLOT);
          pos += 2;
        }
        const int T = passes[pi].j_hi - passes[pi].j_lo + 1;
        for (int i = 0; i < T && ok; ++i, pos += 2) {
          const int kslot = pos % NSLOT;
          if (!mbar_wait(ring_full + kslot, (pos / NSLOT) & 1, abort_flag)) { ok = false; break; }
          const uint32_t kaddr = smem_u32(sRing + kslot * L::kTileBytes);
          for (int a = 0; a < kQT; ++a) {
            // S = Q_a K^T, once the previous S has been copied out
            if (nqk > 0 && !mbar_wait(s_free, (nqk - 1) & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            if constexpr (kQTmem) {
              // A = the rotated query tile in TMEM (8 columns per 16 dimensions)
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t kin = (kk & 3) * 32;   // K step inside a 64-column swizzle block
                umma_ts(tS, tQ + kk * 8, sdesc_sw128(kaddr + (kk >> 2) * kKVBlockBytes + kin, 16, 1024), kIdescQK,
                        kk > 0 ? 1u : 0u);
              }
            } else {
              const uint32_t qaddr = smem_u32(sQ + a * L::kQBytes);
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t kin = (kk & 3) * 32;   // K step inside a 64-column swizzle block
                umma_ss(tS, sdesc_sw128(qaddr + (kk >> 2) * kBlockBytes + kin, 16, 1024),
                        sdesc_sw128(kaddr + (kk >> 2) * kKVBlockBytes + kin, 16, 1024), kIdescQK, kk > 0 ? 1u : 0u);
              }
            }
            umma_commit(s_full + a);
            ++nqk;
          }
          if (!ok) break;
          umma_commit(ring_empty + kslot);
          if (i == T - 1 && pi + 1 < npass) umma_commit(q_free);   // last read of this pass's Q
        }
      }
    }
  } else if (warp >= SH::kWarpPV) {
    // ------------------------------------- MMA: PV of tile warp - kWarpPV
    if constexpr (kQT == 2) reg_dealloc<kProducerRegs>();
    if (lane == 0) {
      const int a = warp - SH::kWarpPV;
      int pos = 0, g = 0;
      bool ok = true;
      for (int pi = 0; pi < npass && ok; ++pi) {
        if constexpr (kQTmem) pos += 2;   // the query tile's two ring positions
        const int T = passes[pi].j_hi - passes[pi].j_lo + 1;
        for (int i = 0; i < T && ok; ++i, ++g, pos += 2) {
          const int vpos = pos + 1, vslot = vpos % NSLOT;
          if (!mbar_wait(ring_full + vslot, (vpos / NSLOT) & 1, abort_flag)) { ok = false; break; }
          // O_a += P_a V once P_a is stored (and, for a later pass, once the
          // previous pass's partial has been read out of O_a)
          if (!mbar_wait(p_full + a, g & 1, abort_flag)) { ok = false; break; }
          if (i == 0 && pi > 0 && !mbar_wait(o_free + a, (pi - 1) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t vaddr = smem_u32(sRing + vslot * L::kTileBytes);
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk) {
            const uint64_t bdesc = sdesc_sw128(vaddr + kk * 2048, kKVBlockBytes, 1024);
            umma_ts(tO + a * D, tP + a * 64 + kk * 8, bdesc, kIdescPV, (kk > 0 || i > 0) ? 1u : 0u);
          }
          umma_commit(o_done + a);
          umma_commit(ring_empty + vslot);   // one of the V slot's two releases
        }
      }
    }
  } else {
    // -------------------------------------------------------------- softmax
    if constexpr (kQT == 2) reg_alloc<kSoftmaxRegs>();
    const int a = warp >> 2;                 // query tile of this warpgroup
    const int row = tid & (kBM - 1);         // TMEM lane == row in the tile
    const int qa0 = q0 + a * kBM;
    const int t = qa0 + row;
    const bool row_ok = t < p.S;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tSw = tS + lane_off;
    const uint32_t tPa = tP + a * 64 + lane_off;
    const uint32_t tOa = tO + a * D + lane_off;
    uint8_t* sQa = sQ + a * L::kQBytes;
    // waits are made warp-uniform so the warp-collective TMEM accesses that
    // follow are always executed by all 32 lanes together
    auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
    };
    const float sl2 = p.scale_log2;
    const bool bif = p.kind == kBifocal;
    float rem_lg = -INFINITY;                // log2-sum-exp of the remote partial (bifocal)
    float* orow = p.out + ((static_cast<size_t>(b) * p.S + (row_ok ? t : 0)) * p.Hq + h) * D;
    bool ok = true;
    int g = 0;
    int qpos = 0;                            // D = 256: ring position of the pass's query tile
    for (int pi = 0; pi < npass && ok; ++pi) {
      const PassDesc ps = passes[pi];
      // ---- rotate this row of the staged query tile (Periodic RoPE §3.1
      // Eq. 2 at the pass's positions)
      if constexpr (kQTmem) {
        // the tile sits in two adjacent ring slots; the rotated row goes to
        // TMEM lane `row` (column c = dimensions 2c, 2c+1), 32 columns per
        // store, once the previous pass's QK^T has read the TMEM tile
        const int qslot = qpos % NSLOT;
        if (!wwait(ring_full + qslot, (qpos / NSLOT) & 1) ||
            !wwait(ring_full + qslot + 1, ((qpos + 1) / NSLOT) & 1)) { ok = false; break; }
        if (pi > 0 && !wwait(q_free, (pi - 1) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint8_t* sq = sRing + qslot * L::kTileBytes;
        const float2* tab = ps.sel ? p.tab1 : p.tab0;
        const float4* tr =
            tab != nullptr ? reinterpret_cast<const float4*>(tab + static_cast<size_t>(row_ok ? t : 0) * (D / 2))
                           : nullptr;
        for (int c0 = 0; c0 < D / 8; c0 += 8) {
          uint32_t w[32];
#pragma unroll
          for (int cc = 0; cc < 8; ++cc) {
            const int c = c0 + cc;
            const int off = (c >> 3) * kBlockBytes + row * 128 + (((c & 7) ^ (row & 7)) << 4);
            const uint4 x = *reinterpret_cast<const uint4*>(sq + off);
            const uint32_t xw[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) w[4 * cc + e] = xw[e];
            if (tr != nullptr && row_ok) {
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const float4 cs = __ldg(tr + c * 2 + e);   // pairs 4c+2e, 4c+2e+1
                float a0, a1;
                rot_pair(bf16lo(xw[2 * e]), bf16hi(xw[2 * e]), cs.x, cs.y, a0, a1);
                w[4 * cc + 2 * e] = pack_bf16x2(a0, a1);
                rot_pair(bf16lo(xw[2 * e + 1]), bf16hi(xw[2 * e + 1]), cs.z, cs.w, a0, a1);
                w[4 * cc + 2 * e + 1] = pack_bf16x2(a0, a1);
              }
            }
          }
          tmem_st32(tQ + lane_off + c0 * 4, w);
        }
        tmem_st_wait();
        // this thread's reads of the two slots are done before the next TMA
        // writes them: the QK issuer hands the slots back once all 128
        // softmax threads have arrived here
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(q_ready + a);
        qpos += 2 + 2 * (ps.j_hi - ps.j_lo + 1);
      }
      if (!kQTmem && !wwait(q_full, pi & 1)) { ok = false; break; }
      if (!kQTmem && p.tab0 != nullptr) {
        const float2* tab = ps.sel ? p.tab1 : p.tab0;
        const float4* tr = reinterpret_cast<const float4*>(tab + static_cast<size_t>(row_ok ? t : 0) * (D / 2));
#pragma unroll 4
        for (int c = 0; c < D / 8; ++c) {
          const int off = (c >> 3) * kBlockBytes + row * 128 + (((c & 7) ^ (row & 7)) << 4);
          uint4* src = reinterpret_cast<uint4*>(sQa + off);
          if (row_ok) {
            const uint4 x = *src;
            const uint32_t xw[4] = {x.x, x.y, x.z, x.w};
            uint32_t y[4];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const float4 cs = __ldg(tr + c * 2 + e);   // pairs 4c+2e, 4c+2e+1
              float a0, a1;
              rot_pair(bf16lo(xw[2 * e]), bf16hi(xw[2 * e]), cs.x, cs.y, a0, a1);
              y[2 * e] = pack_bf16x2(a0, a1);
              rot_pair(bf16lo(xw[2 * e + 1]), bf16hi(xw[2 * e + 1]), cs.z, cs.w, a0, a1);
              y[2 * e + 1] = pack_bf16x2(a0, a1);
            }
            *src = make_uint4(y[0], y[1], y[2], y[3]);
          }
        }
      }
      if constexpr (!kQTmem) {
        fence_proxy_async_smem();
        mbar_arrive(q_ready + a);
      }

      // ---- key tiles of the pass
      float m = -INFINITY, l = 0.f;
      for (int j = ps.j_lo; j <= ps.j_hi; ++j, ++g) {
        if (!wwait(s_full + a, g & 1)) { ok = false; break; }
        tc_fence_after();
        float s[kBN];
        {
          uint32_t r[kBN];
#pragma unroll
          for (int c = 0; c < kBN / 32; ++c) tmem_ld32(tSw + c * 32, *reinterpret_cast<uint32_t(*)[32]>(r + c * 32));
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < kBN; ++e) s[e] = __uint_as_float(r[e]);
        }
        // S is in registers: the other tile's QK may overwrite it
        tc_fence_before();
        mbar_arrive(s_free);
        const int kv0 = j * kBN;
        const int ta0 = p.q_off + qa0;   // absolute position of the tile's first row
        const bool full = (ta0 - kv0 - (kBN - 1) >= ps.hi_off) && (ta0 + kBM - 1 - kv0 <= ps.lo_off);
        if (!full) {
          const int dbase = p.q_off + t - kv0;  // t - s = dbase - c (absolute t)
#pragma unroll
          for (int c = 0; c < kBN; ++c) {
            const int d = dbase - c;
            if (d < ps.hi_off || d > ps.lo_off) s[c] = -INFINITY;
          }
        }
        // row max: 8 independent chains of 3-input max over columns e + 8k
        float mx8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          float x = fmax3(s[e], s[e + 8], s[e + 16]);
#pragma unroll
          for (int k = 3; k + 1 < kBN / 8; k += 2) x = fmax3(x, s[e + 8 * k], s[e + 8 * k + 8]);
          mx8[e] = fmaxf(x, s[e + kBN - 8]);
        }
        float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                         fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
        mx *= sl2;
        // lazy rescale: move the reference max only when it grows by > 8 (x256)
        const bool need = mx > m + 8.0f;
        const float m_new = need ? mx : m;
        const float alpha = need ? ex2(m - m_new) : 1.0f;
        l *= alpha;
        m = m_new;
        const float mu = (m == -INFINITY) ? 0.f : m;
        const float2 sl2x2 = make_float2(sl2, sl2), nmu2 = make_float2(-mu, -mu);
        float2 lsum[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        // P for the whole row in registers first: the exponentials overlap
        // the previous PV of this tile, which still reads P_a and writes O_a
        uint32_t pk[kBN / 2];
#pragma unroll
        for (int e = 0; e < kBN; e += 2) {
          const float2 x = __ffma2_rn(make_float2(s[e], s[e + 1]), sl2x2, nmu2);
          const float2 pp = make_float2(ex2(x.x), ex2(x.y));
          lsum[(e >> 1) & 1] = __fadd2_rn(lsum[(e >> 1) & 1], pp);
          pk[e >> 1] = pack_bf16x2(pp.x, pp.y);
        }
        l += (lsum[0].x + lsum[0].y) + (lsum[1].x + lsum[1].y);
        // the previous PV of this tile must have completed before O_a is
        // rescaled or P_a is overwritten
        if (g > 0 && !wwait(o_done + a, (g - 1) & 1)) { ok = false; break; }
        tc_fence_after();
        if (j != ps.j_lo && __any_sync(0xffffffffu, need)) {
          uint32_t r[32];
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            tmem_ld32(tOa + c * 32, r);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
            tmem_st32(tOa + c * 32, r);
          }
        }
#pragma unroll
        for (int c = 0; c < kBN / 32; ++c) tmem_st16(tPa + c * 16, *reinterpret_cast<const uint32_t(*)[16]>(pk + c * 16));
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(p_full + a);
      }
      if (!ok) break;

      // ---- pass epilogue: wait for the last PV of this tile
      if (!wwait(o_done + a, (g - 1) & 1)) { ok = false; break; }
      tc_fence_after();
      const bool remote_partial = bif && ps.sel == 1;
      if (remote_partial) {
        // park the normalised remote partial in the output row
        const float c0 = l > 0.f ? 1.0f / l : 0.f;
        rem_lg = l > 0.f ? m + __log2f(l) : -INFINITY;
        uint32_t r0[32];
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          tmem_ld32(tOa + c * 32, r0);
          tmem_ld_wait();
          if (row_ok) {
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              *reinterpret_cast<float4*>(orow + c * 32 + e) =
                  make_float4(__uint_as_float(r0[e]) * c0, __uint_as_float(r0[e + 1]) * c0,
                              __uint_as_float(r0[e + 2]) * c0, __uint_as_float(r0[e + 3]) * c0);
          }
        }
        tc_fence_before();
        mbar_arrive(o_free + a);
      } else {
        // final output: this pass alone, or merged with the remote partial by
        // the Eq. 7 weights W_X = exp(l_X - M)
        const float lg = m + __log2f(l);
        float wl = 1.f, wr = 0.f, lse2 = lg;
        if (bif && rem_lg > -INFINITY) {
          const float M = fmaxf(lg, rem_lg);
          const float el = ex2(lg - M), er = ex2(rem_lg - M);
          wl = el / (el + er);
          wr = er / (el + er);
          lse2 = M + __log2f(el + er);
        }
        const float cl = wl / l;
        uint32_t r0[32];
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          tmem_ld32(tOa + c * 32, r0);
          tmem_ld_wait();
          if (row_ok) {
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
              float4 o = make_float4(__uint_as_float(r0[e]) * cl, __uint_as_float(r0[e + 1]) * cl,
                                     __uint_as_float(r0[e + 2]) * cl, __uint_as_float(r0[e + 3]) * cl);
              if (wr != 0.f) {
                const float4 pr = *reinterpret_cast<const float4*>(orow + c * 32 + e);
                o.x = fmaf(pr.x, wr, o.x);
                o.y = fmaf(pr.y, wr, o.y);
                o.z = fmaf(pr.z, wr, o.z);
                o.w = fmaf(pr.w, wr, o.w);
              }
              // final output: streaming store (evict first), so the 2 GiB of
              // output does not leave L2 full of dirty lines for what runs next
              __stcs(reinterpret_cast<float4*>(orow + c * 32 + e), o);
            }
          }
        }
        if (row_ok) __stcs(p.lse + (static_cast<size_t>(b) * p.Hq + h) * p.S + t, lse2 * 0.69314718055994530942f);
      }
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
