// One decode step over an untouched RoPE key cache (Jet-Long §3.2) on the
// fifth-generation tensor cores, sm_100a, for head_dim 64, 128 and 256.
//
// Split-KV: CTA (split, kv head, batch) owns a contiguous key range of one kv
// head; the grid is one wave. The range streams through shared memory by TMA
// in 128-key tiles (128-byte swizzle, no multicast), K tiles and V tiles in
// rings of their own: K in whole tiles, V in 64-key halves, so a V slot is
// free as soon as the four PV MMAs of its half have read it. Per tile, with
// the GQA group's query heads as the MMA's N dimension (the tensor cores see
// the keys as M = 128 rows):
//   S^T = K' Q^T   tcgen05.mma, A = the K tile (K-major), B = the staged
//                  query rows (K-major), fp32 into TMEM (lane = key);
//   softmax        lane = key: the score of each head, exp2 against a lazily
//                  moved reference maximum per head (one barrier reduction
//                  over the four softmax warps asks whether any score exceeds
//                  it by more than 2^8; only then are the tile maxima
//                  exchanged), P^T (bf16) into shared memory;
//   O^T += V^T P^T tcgen05.mma, A = the V tile read MN-major (the head_dim
//                  axis as M), B = P^T, fp32 accumulator in TMEM (lane = one
//                  output dimension).
// The staged query rows are R(p(t)) q for the kind's own position of the query
// token t = n - 1 (rows 0..GP-1) and, for the bifocal map, R(f(t)) q (rows
// GP..2 GP-1), both rotated from the raw query with exact angles in fp32 and
// rounded to bf16. Local keys use the first set as stored in the cache. Remote
// keys k ((n-1) - k > w0) are read through the correction of Eq. 6: the
// rotation warps turn each remote key of the staged K tile in place by
// R(f(k) - k) = R(-u(k)), u(k) = k - floor(k/G), before the MMA reads it. A
// thread of those warps owns one 16-byte chunk (four rotation pairs) of
// every STEP-th row: the (cos, sin) of -u(k) theta_i is advanced row to row,
// and on from one tile to the next, by one of two fixed rotations (u grows by
// STEP - STEP/G, or one less when a group boundary is crossed), and seeded
// exactly every few tiles.
// Every angle is an integer position times theta_i taken from theta_i's
// fraction of a turn in 64-bit fixed point, so it is exact modulo a turn
// before the fp32 sincospi.
//
// Warps: 0-3 softmax (TMEM lanes 0-127), 4-11 key rotation, 12 and 13 TMA
// producers of the K ring and the V ring, 14 QK issuer (one thread; TMEM
// allocation), 15 PV issuer (one thread); all of them stage the query. After the key
// range each CTA writes (O, m, l) of its split, and the last CTA of a (batch,
// kv head) to arrive merges all splits in split order.
#pragma once

#include <type_traits>

#include "common.cuh"
#include "decode_sm100.cuh"
#include "posmap.cuh"

namespace ropeattn {

constexpr int kTcKeys = 128;      // keys per stage (the MMA's M)
constexpr int kTcRotThreads = 256;   // key-rotation warps 4-11
constexpr int kTcThreads = 128 + kTcRotThreads + 128;   // 16 warps
constexpr int kTcWarpTmaK = 12;   // K tile producer
constexpr int kTcWarpTmaV = 13;   // V tile producer
constexpr int kTcWarpQK = 14;     // QK^T issuer (and TMEM allocation)
constexpr int kTcWarpPV = 15;     // PV issuer
constexpr int kTcReseed = 8;      // tiles between exact re-seeds of the rotation phasor
constexpr int kTcNP = 16;         // N of the PV MMA: query heads of the group, padded
constexpr int kTcMaxSplits = 256;   // key-range splits per (batch, kv head), at most

template <int D, int GP, int ROT>
struct DecodeTcShape {
  static constexpr int kRows = ROT ? 2 * GP : GP;          // staged query rows
  static constexpr int NB = kRows <= 16 ? 16 : 32;           // N of the QK MMA
  // A K slot is busy from its load through the rotation and the QK MMA; a V
  // half from its load through its PV MMAs. Each ring must cover the DRAM
  // latency under load (~4000 cycles) plus that work at the HBM rate, with
  // the SM clock as low as the power cap takes it: four K tiles and five V
  // halves at head_dim 128 (208 KiB), seven and twelve at 64; at 256 a tile
  // carries twice the bytes (so twice the time at the HBM rate) and two K
  // tiles and two V halves fill the same space (192 KiB).
  static constexpr int kKSlots = D == 256 ? 2 : (D == 128 ? 4 : 7);      // K ring: whole tiles
  static constexpr int kVHalves = D == 256 ? 2 : (D == 128 ? 5 : 12);    // V ring: 64-key halves
  static constexpr int kMB = D > 128 ? D / 128 : 1;          // O^T blocks of 128 output dimensions
  static constexpr int kHalfKeys = kTcKeys / 2;
  static constexpr int kBlk = kTcKeys * 128;                 // one 64-column swizzle block of a K tile
  static constexpr int kBlkH = kHalfKeys * 128;              // the same block of a V half
  static constexpr int kTileBytes = kTcKeys * D * 2;         // K tile
  static constexpr int kHalfBytes = kHalfKeys * D * 2;       // V half
  static constexpr int kV = 0;                               // V ring, then the K ring
  static constexpr int kK = kVHalves * kHalfBytes;
  static constexpr int kQ = kK + kKSlots * kTileBytes;       // [D/64][NB rows][128 B]
  static constexpr int kQBytes = (D / 64) * NB * 128;
  static constexpr int kP = kQ + kQBytes;                    // [2 bufs][2 key blocks][kTcNP rows][128 B]
  static constexpr int kPBuf = 2 * kTcNP * 128;
  static constexpr int kRed = kP + 2 * kPBuf;                // [4 warps][GP] tile maxima, then [4][GP] sums
  static constexpr int kBar = kRed + 2 * 4 * GP * 4 + 64;
  // kfull, rot, kempty [kKSlots each]; vfull, vempty [kVHalves each];
  // s_full, s_free, p_full, pv_done [2 each]
  static constexpr int kNumBars = 3 * kKSlots + 2 * kVHalves + 8;
  static constexpr int kMisc = kBar + kNumBars * 8;          // tmem base, abort flag, last flag
  static constexpr int kTotal = kMisc + 16;
  static constexpr int kAlloc = kTotal + 1024;               // slack to align the base to 1024
  static constexpr uint32_t kTmemCols = (2 * NB + kMB * kTcNP) <= 64 ? 64 : 128;
  static_assert(GP <= 16, "query heads per kv head: at most 16");
  static_assert(kK % 1024 == 0 && kQ % 1024 == 0 && kP % 1024 == 0 && kPBuf % 1024 == 0 &&
                    (NB * 128) % 1024 == 0 && kHalfBytes % 1024 == 0,
                "swizzled operand tiles start on 1024-byte boundaries");
  // the merge of the splits stages (m, l) of every split of the group in the
  // (then idle) V ring
  static_assert(kK >= kTcMaxSplits * 16 * 8, "the V ring holds (m, l) of every split of a 16-head group");
  static_assert(kAlloc <= 227 * 1024, "shared memory");
};

// one ring slot: kCB boxes of 64 columns x the slot's keys, from key row `row`
template <int kCB>
__device__ __forceinline__ void dec_tile_load(uint8_t* dst, int blk_bytes, int bytes, const CUtensorMap* map,
                                              uint64_t* full, int hkv, int row, int b) {
  mbar_arrive_expect_tx(full, bytes);
#pragma unroll
  for (int cb = 0; cb < kCB; ++cb) tma_load_4d(dst + cb * blk_bytes, map, full, cb * 64, hkv, row, b);
}

// byte offset of element (row, col) of a K-major operand tile stored as
// 64-column blocks of rows x 128 bytes with the 128-byte swizzle
__device__ __forceinline__ int sw128_off(int row, int col, int block_bytes) {
  const int c = (col & 63) >> 3;
  return (col >> 6) * block_bytes + row * 128 + ((c ^ (row & 7)) << 4) + (col & 7) * 2;
}

template <int D, int GP, int ROT>
__global__ void __launch_bounds__(kTcThreads, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const DecodeParams p) {
  using L = DecodeTcShape<D, GP, ROT>;
  constexpr int NK = L::kKSlots;
  constexpr int NVH = L::kVHalves;
  constexpr int NB = L::NB;
  constexpr int kMB = L::kMB;
  constexpr int kCB = D / 64;
  constexpr uint32_t kIdescQK = idesc_bf16_f32(kTcKeys, NB, false, false);
  constexpr uint32_t kIdescPV = idesc_bf16_f32(128, kTcNP, false, true);   // A = V^T read MN-major

  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, by pointer arithmetic on the shared array so the
  // compiler keeps shared-memory (not generic) loads and stores
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sQ = smem + L::kQ;
  uint8_t* sP = smem + L::kP;
  float* red = reinterpret_cast<float*>(smem + L::kRed);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* kfull = bars;            // [NK] K tile landed
  uint64_t* rot = kfull + NK;        // [NK] remote keys of the K tile rotated
  uint64_t* kempty = rot + NK;       // [NK] K tile read by its QK
  uint64_t* vfull = kempty + NK;     // [NVH] V half landed
  uint64_t* vempty = vfull + NVH;    // [NVH] V half read by its PV MMAs
  uint64_t* s_full = vempty + NVH;   // [2]
  uint64_t* s_free = s_full + 2;     // [2]
  uint64_t* p_full = s_free + 2;     // [2]
  uint64_t* pv_done = p_full + 2;    // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  volatile int* last_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 8);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int split = blockIdx.x;
  const int hkv = blockIdx.y;
  const int b = blockIdx.z;

  const int kb = min(p.n, p.k_begin + split * p.keys_per_split);
  const int ke = min(p.n, kb + p.keys_per_split);
  const int ntile = (ke - kb + kTcKeys - 1) / kTcKeys;
  const int t_q = p.n - 1;   // query position index
  const int grp = p.Hq / p.Hkv;   // query heads of the group (<= GP; the rest are zero rows)
  // remote keys [kb, kr_end) come first: the tiles that hold any are a prefix
  const int kr_end = ROT ? min(p.k_local, ke) : kb;
  const int nrot = kr_end > kb ? (kr_end - kb + kTcKeys - 1) / kTcKeys : 0;

  if (tid == 0) {
    for (int i = 0; i < NK; ++i) {
      mbar_init(kfull + i, 1);
      mbar_init(rot + i, kTcRotThreads);
      mbar_init(kempty + i, 1);
    }
    for (int i = 0; i < NVH; ++i) {
      mbar_init(vfull + i, 1);
      mbar_init(vempty + i, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(s_full + a, 1);
      mbar_init(s_free + a, 128);
      mbar_init(p_full + a, 128);
      mbar_init(pv_done + a, 1);
    }
    *abort_flag = 0;
    *last_flag = 0;
    mbar_fence_init();
  }
  if (warp == kTcWarpQK) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  // zero the staged query rows and both P^T buffers (rows beyond the group
  // stay zero), then stage the rotated query rows
  for (int i = tid; i < (L::kQBytes + 2 * L::kPBuf) / 16; i += kTcThreads)
    reinterpret_cast<uint4*>(sQ)[i] = make_uint4(0u, 0u, 0u, 0u);
  __syncthreads();
  // the query words of this thread's staging items (at most two: GP <= 16)
  constexpr int kQItems = (GP * (D / 2) + kTcThreads - 1) / kTcThreads;
  uint32_t qw[kQItems];
#pragma unroll
  for (int u = 0; u < kQItems; ++u) {
    const int i = tid + u * kTcThreads;
    if (i < grp * (D / 2)) {
      const int hq = hkv * grp + i / (D / 2);
      qw[u] = __ldg(reinterpret_cast<const uint32_t*>(p.q + (static_cast<size_t>(b) * p.Hq + hq) * D) + i % (D / 2));
    }
  }
  // the first loads of both rings need no free slot: issue them now (after
  // the query loads, which would otherwise queue behind them), so their DRAM
  // latency overlaps the query staging
  const int nhalf = 2 * ntile;
  if (lane == 0 && warp == kTcWarpTmaK) {
    tma_prefetch_desc(&tmK);
    for (int t = 0; t < min(NK, ntile); ++t)
      dec_tile_load<kCB>(smem + L::kK + (t % NK) * L::kTileBytes, L::kBlk, L::kTileBytes, &tmK, kfull + t % NK,
                         hkv, kb + t * kTcKeys, b);
  } else if (lane == 0 && warp == kTcWarpTmaV) {
    tma_prefetch_desc(&tmV);
    for (int j = 0; j < min(NVH, nhalf); ++j)
      dec_tile_load<kCB>(smem + L::kV + (j % NVH) * L::kHalfBytes, L::kBlkH, L::kHalfBytes, &tmV, vfull + j % NVH,
                         hkv, kb + j * L::kHalfKeys, b);
  }
#pragma unroll
  for (int u = 0; u < kQItems; ++u) {
    const int i = tid + u * kTcThreads;
    if (i >= grp * (D / 2)) continue;
    const int gi = i / (D / 2), pr = i % (D / 2);
    const uint32_t xw = qw[u];
    const float x0 = bf16lo(xw), x1 = bf16hi(xw);
    uint32_t yl = xw;
    if (p.m.kind != kNope) {
      const float2 cs = turn_cs(pos_primary(p.m, t_q), p.turns[pr]);
      float y0, y1;
      rot_pair(x0, x1, cs.x, cs.y, y0, y1);
      yl = pack_bf16x2(y0, y1);
    }
    *reinterpret_cast<uint32_t*>(sQ + sw128_off(gi, 2 * pr, NB * 128)) = yl;
    if constexpr (ROT != 0) {
      const float2 cs = turn_cs(pos_remote(p.m, t_q), p.turns[pr]);
      float y0, y1;
      rot_pair(x0, x1, cs.x, cs.y, y0, y1);
      *reinterpret_cast<uint32_t*>(sQ + sw128_off(GP + gi, 2 * pr, NB * 128)) = pack_bf16x2(y0, y1);
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem;              // S^T buffers at [0, NB) and [NB, 2 NB)
  const uint32_t tO = tmem + 2 * NB;     // O^T, kTcNP columns per block of 128 dimensions

  float l_fin[GP];                      // softmax threads: per-thread sums, reduced at the end
  float m_fin[GP];
#pragma unroll
  for (int gi = 0; gi < GP; ++gi) {
    l_fin[gi] = 0.f;
    m_fin[gi] = -INFINITY;
  }
  uint32_t o_fin[kMB][kTcNP];

  if (warp == kTcWarpTmaK || warp == kTcWarpTmaV) {
    // -------------------------------------------------------- TMA producers
    // K tiles and V halves stream through rings of their own: a K slot is
    // free once its QK has read it, a V half once its PV MMAs have, so K
    // tiles run ahead of the rotation and the values of a tile are fetched
    // while it is scored
    if (lane == 0) {
      if (warp == kTcWarpTmaK) {
        for (int t = NK; t < ntile; ++t) {
          if (!mbar_wait(kempty + t % NK, ((t / NK) - 1) & 1, abort_flag)) break;
          dec_tile_load<kCB>(smem + L::kK + (t % NK) * L::kTileBytes, L::kBlk, L::kTileBytes, &tmK, kfull + t % NK,
                             hkv, kb + t * kTcKeys, b);
        }
      } else {
        for (int j = NVH; j < nhalf; ++j) {
          if (!mbar_wait(vempty + j % NVH, ((j / NVH) - 1) & 1, abort_flag)) break;
          dec_tile_load<kCB>(smem + L::kV + (j % NVH) * L::kHalfBytes, L::kBlkH, L::kHalfBytes, &tmV, vfull + j % NVH,
                             hkv, kb + j * L::kHalfKeys, b);
        }
      }
    }
  } else if (warp == kTcWarpQK) {
    // -------------------------------------------------------- MMA: S^T = K Q^T
    if (lane == 0) {
      const uint32_t qaddr = smem_u32(sQ);
      for (int t = 0; t < ntile; ++t) {
        const int s = t % NK;
        if (!mbar_wait(t < nrot ? rot + s : kfull + s, (t / NK) & 1, abort_flag)) break;
        if (t >= 2 && !mbar_wait(s_free + (t & 1), ((t >> 1) - 1) & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t kaddr = smem_u32(smem + L::kK + s * L::kTileBytes);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t kin = (kk & 3) * 32;   // K step inside a 64-column swizzle block
          umma_ss(tS + (t & 1) * NB, sdesc_sw128(kaddr + (kk >> 2) * L::kBlk + kin, 16, 1024),
                  sdesc_sw128(qaddr + (kk >> 2) * (NB * 128) + kin, 16, 1024), kIdescQK, kk > 0 ? 1u : 0u);
        }
        umma_commit(s_full + (t & 1));
        umma_commit(kempty + s);
      }
    }
  } else if (warp == kTcWarpPV) {
    // ------------------------------------------------------ MMA: O^T += V^T P^T
    if (lane == 0) {
      for (int t = 0; t < ntile; ++t) {
        if (!mbar_wait(p_full + (t & 1), (t >> 1) & 1, abort_flag)) break;
        const uint32_t paddr = smem_u32(sP + (t & 1) * L::kPBuf);
        bool okv = true;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int j = 2 * t + h;
          const int s = j % NVH;
          if (!mbar_wait(vfull + s, (j / NVH) & 1, abort_flag)) { okv = false; break; }
          tc_fence_after();
          const uint32_t vaddr = smem_u32(smem + L::kV + s * L::kHalfBytes);
          // M = 128 output dimensions per MMA (two 64-column blocks of the
          // half, one O^T block); for D = 64 the upper 64 rows read the 8 KiB
          // that follow the V half (the next half, or the K ring) and land in
          // TMEM lanes nobody reads
#pragma unroll
          for (int mb = 0; mb < kMB; ++mb)
#pragma unroll
            for (int kq = 0; kq < L::kHalfKeys / 16; ++kq) {
              const int kk = h * (L::kHalfKeys / 16) + kq;
              umma_ss(tO + mb * kTcNP, sdesc_sw128(vaddr + 2 * mb * L::kBlkH + kq * 2048, L::kBlkH, 1024),
                      sdesc_sw128(paddr + (kk >> 2) * (kTcNP * 128) + (kk & 3) * 32, 16, 1024), kIdescPV,
                      (t > 0 || kk > 0) ? 1u : 0u);
            }
          umma_commit(vempty + s);
        }
        if (!okv) break;
        umma_commit(pv_done + (t & 1));
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------- rotation of remote keys
    if constexpr (ROT != 0) {
      constexpr int CPR = D / 8;              // 16-byte chunks per row
      constexpr int STEP = kTcRotThreads / CPR;   // rows between a thread's rows (16 or 32)
      constexpr int NR = kTcKeys / STEP;      // rows per thread per tile (8 or 4)
      const int id = tid - 128;
      const int c = id % CPR, rg = id / CPR;
      const int G = p.m.G;
      const int stepq = STEP / G, stepr = STEP % G;
      // the two row-to-row advances of u: STEP - stepq, and one less after a
      // group boundary; (cos, sin, -sin) of -du theta for the thread's pairs
      float2 MC[2][2], MS[2][2], MNS[2][2];   // [advance][pair pack] (pairs 4c+2j, 4c+2j+1)
#pragma unroll
      for (int e = 0; e < 2; ++e)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int du = STEP - stepq - e;
          const float2 x = turn_cs(-du, p.turns[4 * c + 2 * j]);
          const float2 y = turn_cs(-du, p.turns[4 * c + 2 * j + 1]);
          MC[e][j] = f2(x.x, y.x);
          MS[e][j] = f2(x.y, y.y);
          MNS[e][j] = f2(-x.y, -y.y);
        }
      // The thread's rows of consecutive tiles are STEP apart across the tile
      // boundary too, so the phasor (cos, sin)(-u(k) theta) carries from one
      // tile to the next; it is re-seeded exactly every kTcReseed tiles.
      int k = kb + rg;                        // key of the thread's next row
      int rem = 0;                            // k mod G
      float2 C[2], S[2];
      auto seed = [&]() {
        const int qd = k / G;
        rem = k - qd * G;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const float2 x = turn_cs(-(k - qd), p.turns[4 * c + 2 * j]);
          const float2 y = turn_cs(-(k - qd), p.turns[4 * c + 2 * j + 1]);
          C[j] = f2(x.x, y.x);
          S[j] = f2(x.y, y.y);
        }
      };
      auto mult = [&](int e) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const float2 cn = fma2(C[j], MC[e][j], mul2(S[j], MNS[e][j]));
          const float2 sn = fma2(C[j], MS[e][j], mul2(S[j], MC[e][j]));
          C[j] = cn;
          S[j] = sn;
        }
      };
      // (x0 c - x1 s, x0 s + x1 c) on the chunk's four pairs, (c, s) = (cos, sin)(-u theta)
      auto turn = [&](uint4 x) -> uint4 {
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
        uint32_t y[4];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const float2 X0 = f2(bf16lo(w[2 * j]), bf16lo(w[2 * j + 1]));
          const float2 X1 = f2(bf16hi(w[2 * j]), bf16hi(w[2 * j + 1]));
          const float2 Y0 = fma2(neg2(X1), S[j], mul2(X0, C[j]));
          const float2 Y1 = fma2(X0, S[j], mul2(X1, C[j]));
          y[2 * j] = pack_bf16x2(Y0.x, Y1.x);
          y[2 * j + 1] = pack_bf16x2(Y0.y, Y1.y);
        }
        return make_uint4(y[0], y[1], y[2], y[3]);
      };
      // u(k + STEP) - u(k) = STEP - (floor((k + STEP)/G) - floor(k/G)); the
      // advance without a group-boundary carry when G divides STEP (FAST),
      // else the carried one picked by selects, so a tile is straight-line code
      auto advance = [&](auto fast_tag) {
        constexpr bool FAST = decltype(fast_tag)::value;
        k += STEP;
        if constexpr (FAST) {
          mult(0);
        } else {
          rem += stepr;
          const bool e = rem >= G;
          rem -= e ? G : 0;
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const float2 mc = e ? MC[1][j] : MC[0][j];
            const float2 ms = e ? MS[1][j] : MS[0][j];
            const float2 mns = e ? MNS[1][j] : MNS[0][j];
            const float2 cn = fma2(C[j], mc, mul2(S[j], mns));
            const float2 sn = fma2(C[j], ms, mul2(S[j], mc));
            C[j] = cn;
            S[j] = sn;
          }
        }
      };
      // every row of the tile is remote: all loads first, then rotate and store
      auto tile_full = [&](uint8_t* kt, auto fast_tag) {
        uint4 x[NR];
#pragma unroll
        for (int m = 0; m < NR; ++m) {
          const int r = rg + STEP * m;
          x[m] = *reinterpret_cast<const uint4*>(kt + r * 128 + (((c & 7) ^ (r & 7)) << 4));
        }
#pragma unroll
        for (int m = 0; m < NR; ++m) {
          x[m] = turn(x[m]);
          advance(fast_tag);
        }
#pragma unroll
        for (int m = 0; m < NR; ++m) {
          const int r = rg + STEP * m;
          *reinterpret_cast<uint4*>(kt + r * 128 + (((c & 7) ^ (r & 7)) << 4)) = x[m];
        }
      };
      for (int t = 0; t < nrot; ++t) {
        const int s = t % NK;
        if (!__all_sync(0xffffffffu, mbar_wait(kfull + s, (t / NK) & 1, abort_flag))) break;
        if (t % kTcReseed == 0) seed();
        uint8_t* kt = smem + L::kK + s * L::kTileBytes + (c >> 3) * L::kBlk;
        const int k0 = kb + t * kTcKeys;
        if (k0 + kTcKeys <= kr_end) {
          if (stepr == 0) {
            tile_full(kt, std::true_type{});
          } else {
            tile_full(kt, std::false_type{});
          }
        } else {
          // the tile reaching the local window (or the end of the split)
#pragma unroll
          for (int m = 0; m < NR; ++m) {
            const int r = rg + STEP * m;
            if (k < kr_end) {
              uint4* a = reinterpret_cast<uint4*>(kt + r * 128 + (((c & 7) ^ (r & 7)) << 4));
              *a = turn(*a);
            }
            advance(std::false_type{});
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(rot + s);
      }
    }
  } else {
    // -------------------------------------------------------------- softmax
    const int r = tid;                                   // key row of a tile; O^T row (dimension)
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const float sl2 = p.scale_log2;
    auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
    };
    float m_run[GP], l_thr[GP];
#pragma unroll
    for (int gi = 0; gi < GP; ++gi) {
      m_run[gi] = -INFINITY;
      l_thr[gi] = 0.f;
    }
    bool ok = true;
    for (int t = 0; t < ntile; ++t) {
      const int k = kb + t * kTcKeys + r;
      // a failed wait does not leave the loop on its own: it is reduced with
      // the other softmax warps at the tile's barrier below, so all four
      // leave together and none waits at a barrier the others have left
      const bool okw = ok && wwait(s_full + (t & 1), (t >> 1) & 1);
      float sc[GP];
      bool raise = false;   // a score above the reference maximum by more than 8 (x256)
      if (okw) {
        tc_fence_after();
        uint32_t sv[NB];
        if constexpr (NB == 16) {
          tmem_ld16(tS + (t & 1) * NB + lane_off, *reinterpret_cast<uint32_t(*)[16]>(sv));
        } else {
          tmem_ld32(tS + (t & 1) * NB + lane_off, *reinterpret_cast<uint32_t(*)[32]>(sv));
        }
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(s_free + (t & 1));
        const bool valid = k < ke;
        const bool remote = ROT != 0 && k < p.k_local;
#pragma unroll
        for (int gi = 0; gi < GP; ++gi) {
          const uint32_t raw = remote ? sv[(ROT != 0 ? GP : 0) + gi] : sv[gi];
          sc[gi] = valid ? __uint_as_float(raw) * sl2 : -INFINITY;
          raise |= sc[gi] > m_run[gi] + 8.0f;
        }
      } else {
#pragma unroll
        for (int gi = 0; gi < GP; ++gi) sc[gi] = -INFINITY;
      }
      // lazy rescale: the reference maximum of a head moves only when the
      // tile's maximum exceeds it by more than 8. Whether any head must move
      // (or any wait failed) is one barrier reduction over the 128 softmax
      // threads; only then are the tile maxima exchanged
      bool need_any = false;
      float corr[GP];
#pragma unroll
      for (int gi = 0; gi < GP; ++gi) corr[gi] = 1.0f;
      if (bar_red_or(1, 128, raise || !okw)) {
        if (bar_red_or(1, 128, !okw)) { ok = false; break; }
        float wm[GP];
#pragma unroll
        for (int gi = 0; gi < GP; ++gi) wm[gi] = sc[gi];
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1)
#pragma unroll
          for (int gi = 0; gi < GP; ++gi) wm[gi] = fmaxf(wm[gi], __shfl_xor_sync(0xffffffffu, wm[gi], off));
        // one buffer: every thread has read it before any passes the next
        // tile's barrier reduction, and only then is it written again
        if (lane == 0) {
#pragma unroll
          for (int gi = 0; gi < GP; ++gi) red[warp * GP + gi] = wm[gi];
        }
        bar_sync_named(1, 128);
#pragma unroll
        for (int gi = 0; gi < GP; ++gi) {
          const float tmax = fmaxf(fmaxf(red[gi], red[GP + gi]), fmaxf(red[2 * GP + gi], red[3 * GP + gi]));
          const bool need = tmax > m_run[gi] + 8.0f;
          const float m_new = need ? tmax : m_run[gi];
          corr[gi] = need ? ex2(m_run[gi] - m_new) : 1.0f;
          l_thr[gi] *= corr[gi];
          m_run[gi] = m_new;
          need_any |= need;
        }
      }
      uint32_t pb[GP];
#pragma unroll
      for (int gi = 0; gi < GP; ++gi) {
        const float mu = m_run[gi] == -INFINITY ? 0.f : m_run[gi];
        const float pval = ex2(sc[gi] - mu);
        l_thr[gi] += pval;
        pb[gi] = pack_bf16x2(pval, 0.f) & 0xFFFFu;
      }
      // P^T buffer t&1 was last read by PV(t-2); a failed wait skips the
      // rest of the tile and is reduced at the next tile's barrier
      if (t >= 2 && !wwait(pv_done + (t & 1), ((t >> 1) - 1) & 1)) { ok = false; continue; }
      if (t >= 1 && need_any) {
        // rescale O^T (lane r = output dimension r) once PV(t-1) has completed
        if (!wwait(pv_done + ((t - 1) & 1), ((t - 1) >> 1) & 1)) { ok = false; continue; }
        tc_fence_after();
#pragma unroll
        for (int mb = 0; mb < kMB; ++mb) {
          uint32_t o[kTcNP];
          tmem_ld16(tO + mb * kTcNP + lane_off, o);
          tmem_ld_wait();
#pragma unroll
          for (int gi = 0; gi < GP; ++gi) o[gi] = __float_as_uint(__uint_as_float(o[gi]) * corr[gi]);
          tmem_st16(tO + mb * kTcNP + lane_off, o);
        }
        tmem_st_wait();
      }
      uint8_t* pbuf = sP + (t & 1) * L::kPBuf;
#pragma unroll
      for (int gi = 0; gi < GP; ++gi)
        *reinterpret_cast<uint16_t*>(pbuf + sw128_off(gi, r, kTcNP * 128)) = static_cast<uint16_t>(pb[gi]);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full + (t & 1));
    }
    // the last PV has completed: row r of O^T block mb holds this split's
    // unnormalised output of dimension 128 mb + r for every head of the group
    if (ok && ntile > 0 && wwait(pv_done + ((ntile - 1) & 1), ((ntile - 1) >> 1) & 1)) {
      tc_fence_after();
#pragma unroll
      for (int mb = 0; mb < kMB; ++mb) tmem_ld16(tO + mb * kTcNP + lane_off, o_fin[mb]);
      tmem_ld_wait();
    } else {
#pragma unroll
      for (int mb = 0; mb < kMB; ++mb)
#pragma unroll
        for (int i = 0; i < kTcNP; ++i) o_fin[mb][i] = 0u;
    }
#pragma unroll
    for (int gi = 0; gi < GP; ++gi) {
      float l = l_thr[gi];
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
      l_fin[gi] = l;
      m_fin[gi] = m_run[gi];
    }
  }

  // ------------------------------------------------------ split partials
  tc_fence_before();
  __syncthreads();   // every role is done with the ring, TMEM and the reduction buffer
  float* lsum = red;   // [4 warps][GP] sums, then [GP] maxima
  if (warp < 4) {
    if (lane == 0) {
#pragma unroll
      for (int gi = 0; gi < GP; ++gi) {
        lsum[warp * GP + gi] = l_fin[gi];
        if (warp == 0) lsum[4 * GP + gi] = m_fin[gi];   // the reference max, the same in every thread
      }
    }
#pragma unroll
    for (int mb = 0; mb < kMB; ++mb) {
      const int d = mb * 128 + tid;
      if (d < D) {
#pragma unroll
        for (int gi = 0; gi < GP; ++gi) {
          if (gi < grp) {
            const int hq = hkv * grp + gi;
            const size_t pslot = (static_cast<size_t>(b) * p.Hq + hq) * p.nsplit + split;
            p.part_o[pslot * D + d] = __uint_as_float(o_fin[mb][gi]);
          }
        }
      }
    }
  }
  __syncthreads();
  if (tid < grp) {
    const int gi = tid;
    const float l = (lsum[gi] + lsum[GP + gi]) + (lsum[2 * GP + gi] + lsum[3 * GP + gi]);
    const int hq = hkv * grp + gi;
    const size_t pslot = (static_cast<size_t>(b) * p.Hq + hq) * p.nsplit + split;
    p.part_ml[pslot] = make_float2(lsum[4 * GP + gi], l);
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const int prev = atomicAdd(p.counters + b * p.Hkv + hkv, 1);
    *last_flag = (prev == p.nsplit - 1) ? 1 : 0;
  }
  __syncthreads();
  if (*last_flag) {
    // last CTA of this (batch, kv head): merge every split, in split order.
    // The (m, l) of all splits of the group are staged in the idle V ring
    // and turned into the weights exp2(m_s - M) once, so each output element
    // is one pass of independent loads over the splits
    __threadfence();
    const int ns = p.nsplit;
    float2* wml = reinterpret_cast<float2*>(smem + L::kV);   // [grp][ns] (m, l), then (weight, 0)
    float* wtot = reinterpret_cast<float*>(smem + L::kK);   // [grp] (M, L), in the idle K ring
    const size_t gbase = (static_cast<size_t>(b) * p.Hq + hkv * grp) * ns;
    for (int i = tid; i < grp * ns; i += kTcThreads) wml[i] = __ldcg(p.part_ml + gbase + i);
    __syncthreads();
    if (tid < grp) {
      float2* w = wml + tid * ns;
      float M = -INFINITY;
      for (int sp = 0; sp < ns; ++sp)
        if (w[sp].y > 0.f) M = fmaxf(M, w[sp].x);
      float l = 0.f;
      for (int sp = 0; sp < ns; ++sp) {
        const float f = w[sp].y > 0.f ? ex2(w[sp].x - M) : 0.f;
        l = fmaf(w[sp].y, f, l);
        w[sp].x = f;
      }
      wtot[2 * tid] = M;
      wtot[2 * tid + 1] = l;
    }
    __syncthreads();
    for (int idx = tid; idx < grp * D; idx += kTcThreads) {
      const int gi = idx / D, d = idx % D;
      const float2* w = wml + gi * ns;
      const float* po = p.part_o + (gbase + static_cast<size_t>(gi) * ns) * D + d;
      float o = 0.f;
#pragma unroll 8
      for (int sp = 0; sp < ns; ++sp) o = fmaf(__ldcg(po + static_cast<size_t>(sp) * D), w[sp].x, o);
      const int hq = hkv * grp + gi;
      const float M = wtot[2 * gi], l = wtot[2 * gi + 1];
      p.out[(static_cast<size_t>(b) * p.Hq + hq) * D + d] = o / l;
      if (d == 0) p.lse[static_cast<size_t>(b) * p.Hq + hq] = (M + __log2f(l)) * 0.69314718055994530942f;
    }
    if (tid == 0) p.counters[b * p.Hkv + hkv] = 0;
  }
  if (*abort_flag) {
    // let in-flight TMA and MMA work drain before the CTA releases its memory
    const unsigned long long t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 20000000ull) __nanosleep(100000);
  }
  if (warp == kTcWarpQK) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

}  // namespace ropeattn
