// Host side of the ropeattn C ABI: argument checks, workspace layout, TMA
// tensor maps and kernel launches. All kernels live in this translation unit.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "../../include/ropeattn.h"
#include "common.cuh"
#include "cache.cuh"
#include "pairing.cuh"
#include "decode_sm100.cuh"
#include "decode_tc_sm100.cuh"
#include "backward_sm100.cuh"
#include "merge.cuh"
#include "selftest.cuh"
#include "posmap.cuh"
#include "prefill_sm100.cuh"
#include "prep.cuh"

using namespace ropeattn;

namespace {

constexpr int kVersion = 10100;  // 1.1.0: half-split pairing, head_dim 256 prefill
thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(ROPEATTN_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

#define CUDA_TRY(call, what)                 \
  do {                                       \
    cudaError_t _e = (call);                 \
    if (_e != cudaSuccess) return cuda_fail(_e, what); \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// sm_100 check, cached per device
int check_device() {
  static std::mutex mu;
  static int cached[64];  // 0 unknown, 1 ok, -1 bad
  int dev = 0;
  CUDA_TRY(cudaGetDevice(&dev), "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(ROPEATTN_ERR_UNSUPPORTED_DEVICE, "device index %d", dev);
  std::lock_guard<std::mutex> lk(mu);
  if (cached[dev] == 0) {
    int major = 0, minor = 0;
    CUDA_TRY(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev), "cudaDeviceGetAttribute");
    CUDA_TRY(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev), "cudaDeviceGetAttribute");
    cached[dev] = (major == 10 && minor == 0) ? 1 : -1;
    if (cached[dev] < 0)
      return fail(ROPEATTN_ERR_UNSUPPORTED_DEVICE, "device %d is sm_%d%d; this library is built for sm_100a", dev,
                  major, minor);
  }
  if (cached[dev] < 0) return fail(ROPEATTN_ERR_UNSUPPORTED_DEVICE, "device %d is not sm_100", dev);
  return ROPEATTN_OK;
}

// SM count of the current device, looked up once per device
int sm_count() {
  static int cached[64];
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return n;
  if (cached[dev] > 0) return cached[dev];
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  n = n > 0 ? n : 148;
  cached[dev] = n;
  return n;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// TMA map of a 4-D bf16 tensor [d3][d2][d1][d0] (d0 contiguous) with box
// (b0, 1, b2, 1); d2_stride: rows of d2 between consecutive d3 indices (d2
// when 0: a dense tensor; larger for a cache with spare rows).
int make_map(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t d3,
             uint32_t b0, uint32_t b2, bool swizzle128, uint64_t d2_stride = 0) {
  auto fn = encode_fn();
  if (!fn) return fail(ROPEATTN_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t dims[4] = {d0, d1, d2, d3};
  cuuint64_t strides[3] = {d0 * 2, d0 * d1 * 2, d0 * d1 * (d2_stride ? d2_stride : d2) * 2};
  cuuint32_t box[4] = {b0, 1, b2, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(ROPEATTN_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return ROPEATTN_OK;
}

constexpr long long kMaxPos = 0x7fffffffLL;

// Validates the parameter struct for a sequence of length L; fills the
// position map. The kind may be simplified: a bifocal map with G = 1 or with
// every key inside the local window is exactly the standard map (Jet-Long §3:
// the method then gives the base model's attention unchanged).
int check_params(const ropeattn_params* p, long long L, int D, PosMap* m, int* eff_kind) {
  if (!p) return fail(ROPEATTN_ERR_INVALID_ARG, "params is NULL");
  if (p->reserved[0] != 0 || p->reserved[1] != 0)
    return fail(ROPEATTN_ERR_INVALID_ARG, "reserved fields must be 0");
  if (p->pairing != ROPEATTN_PAIR_ADJACENT && p->pairing != ROPEATTN_PAIR_HALF)
    return fail(ROPEATTN_ERR_INVALID_ARG, "pairing must be ROPEATTN_PAIR_ADJACENT or ROPEATTN_PAIR_HALF");
  if (p->fixed_group < 0 || p->fixed_group > (1 << 30) || (p->fixed_group != 0 && p->kind != ROPEATTN_BIFOCAL))
    return fail(ROPEATTN_ERR_INVALID_ARG, "fixed_group must be 0, or in [1, 2^30] for BIFOCAL");
  if (p->kind < ROPEATTN_STANDARD || p->kind > ROPEATTN_BIFOCAL)
    return fail(ROPEATTN_ERR_INVALID_ARG, "unknown kind %d", p->kind);
  if (p->kind != ROPEATTN_NOPE && !(p->rope_base > 1.0 && std::isfinite(p->rope_base)))
    return fail(ROPEATTN_ERR_INVALID_ARG, "rope_base must be a finite number > 1");
  if (!(p->softmax_scale >= 0.0f) || !std::isfinite(p->softmax_scale))
    return fail(ROPEATTN_ERR_INVALID_ARG, "softmax_scale must be >= 0 and finite");
  if (L < 0 || L > kMaxPos) return fail(ROPEATTN_ERR_INVALID_ARG, "sequence length %lld out of range", L);
  *m = PosMap{p->kind, 0, 0, 1, 0, 1};
  *eff_kind = p->kind;
  switch (p->kind) {
    case ROPEATTN_ENDPROMPT:
      if (!(p->interp >= 1.0 && std::isfinite(p->interp)))
        return fail(ROPEATTN_ERR_INVALID_ARG, "interp must be >= 1");
      if (p->seg1_len < 0 || p->term_start < 0 || p->seg1_len > kMaxPos || p->term_start > kMaxPos)
        return fail(ROPEATTN_ERR_INVALID_ARG, "seg1_len and term_start must be in [0, 2^31)");
      if (L > p->seg1_len && p->term_start + (L - 1 - p->seg1_len) > kMaxPos)
        return fail(ROPEATTN_ERR_INVALID_ARG, "terminal positions exceed 2^31-1");
      m->seg1_len = static_cast<int>(p->seg1_len);
      m->term_start = static_cast<int>(p->term_start);
      break;
    case ROPEATTN_PERIODIC:
      if (p->window < 1 || p->window > (1LL << 30)) return fail(ROPEATTN_ERR_INVALID_ARG, "window must be in [1, 2^30]");
      m->window = static_cast<int>(p->window);
      break;
    case ROPEATTN_BIFOCAL: {
      if (p->w0 < 0) return fail(ROPEATTN_ERR_INVALID_ARG, "w0 must be >= 0");
      if (p->fixed_group == 0 && p->w_pretrained < 1)
        return fail(ROPEATTN_ERR_INVALID_ARG, "w_pretrained must be >= 1");
      m->G = p->fixed_group > 0 ? p->fixed_group : group_size(L, p->w_pretrained);
      m->w0 = static_cast<int>(p->w0 < (1LL << 30) ? p->w0 : (1LL << 30));
      if (m->G == 1 || p->w0 >= L - 1) *eff_kind = ROPEATTN_STANDARD;
      break;
    }
    default:
      break;
  }
  (void)D;
  return ROPEATTN_OK;
}

// True when the rotation pairs (i, i + D/2): the query is then permuted to
// adjacent order on entry and keys where they are rotated (pairing.cuh).
bool half_pairing(const ropeattn_params* p) {
  return p->pairing == ROPEATTN_PAIR_HALF && p->kind != ROPEATTN_NOPE;
}

// rows x D bf16 from half-split to adjacent order (pairing.cuh).
int launch_interleave(const void* in, void* out, long long rows, int D, cudaStream_t st) {
  PairInterleaveArgs a{};
  a.in = static_cast<const uint2*>(in);
  a.out = static_cast<uint4*>(out);
  a.rows = rows;
  a.D = D;
  const long long threads = rows * (D / 8);
  pair_interleave_kernel<<<static_cast<unsigned>((threads + 255) / 256), 256, 0, st>>>(a);
  CUDA_TRY(cudaGetLastError(), "pair_interleave launch");
  return ROPEATTN_OK;
}

void fill_theta(const ropeattn_params* p, int D, double* theta) {
  const double s = p->kind == ROPEATTN_ENDPROMPT ? p->interp : 1.0;
  for (int i = 0; i < D / 2; ++i) theta[i] = std::pow(p->rope_base, -2.0 * i / D) / s;
}

// theta_i / (2 pi) modulo 1 in 64-bit fixed point (units of 2^-64 turn),
// computed in long double from the double theta_i of fill_theta. The last
// few results are kept per thread (a decode step calls this every time, and
// the long-double arithmetic costs tens of microseconds of host time).
void fill_turns(const ropeattn_params* p, int D, unsigned long long* turns) {
  struct Entry {
    double base, s;
    int D;
    unsigned long long turns[kMaxPairs];
  };
  constexpr int kCache = 4;
  thread_local Entry cache[kCache];
  thread_local int used = 0, next = 0;
  const double s = p->kind == ROPEATTN_ENDPROMPT ? p->interp : 1.0;
  for (int e = 0; e < used; ++e) {
    if (cache[e].base == p->rope_base && cache[e].s == s && cache[e].D == D) {
      std::memcpy(turns, cache[e].turns, sizeof(unsigned long long) * (D / 2));
      return;
    }
  }
  double theta[kMaxPairs];
  fill_theta(p, D, theta);
  const long double two_pi = 2.0L * std::acos(-1.0L);
  for (int i = 0; i < D / 2; ++i) {
    long double f = std::fmod(static_cast<long double>(theta[i]) / two_pi, 1.0L);
    if (f < 0) f += 1.0L;
    const long double r = std::floor(std::ldexp(f, 64) + 0.5L);
    turns[i] = r >= 18446744073709551616.0L ? 0ull : static_cast<unsigned long long>(r);   // 2^64 wraps to 0
  }
  Entry& slot = cache[next];
  slot.base = p->rope_base;
  slot.s = s;
  slot.D = D;
  std::memcpy(slot.turns, turns, sizeof(unsigned long long) * (D / 2));
  next = (next + 1) % kCache;
  if (used < kCache) ++used;
}

float scale_log2(const ropeattn_params* p, int D) {
  const double sc = p->softmax_scale > 0.0f ? static_cast<double>(p->softmax_scale) : 1.0 / std::sqrt(double(D));
  return static_cast<float>(sc * 1.4426950408889634074);
}

// Shapes every entry point accepts: D = 64, 128 or 256 (the prefill runs
// D = 256 with one query tile per CTA, PrefillShape).
int check_shapes(long long B, long long S, int Hq, int Hkv, int D) {
  if (B < 0 || S < 0) return fail(ROPEATTN_ERR_INVALID_ARG, "B and S must be >= 0");
  if (D != 64 && D != 128 && D != 256)
    return fail(ROPEATTN_ERR_INVALID_ARG, "D must be 64, 128 or 256 (got %d)", D);
  if (Hq < 1 || Hkv < 1 || Hq % Hkv != 0)
    return fail(ROPEATTN_ERR_INVALID_ARG, "need Hq >= 1, Hkv >= 1 and Hq %% Hkv == 0 (Hq=%d Hkv=%d)", Hq, Hkv);
  if (S > kMaxPos || B > 65535 || Hq > 65535) return fail(ROPEATTN_ERR_INVALID_ARG, "shape too large");
  return ROPEATTN_OK;
}

struct PrefillLayout {
  int nmaps;
  bool half;
  size_t krot_bytes, tab_bytes, total;
  size_t off_krot[2], off_tab[2], off_q;
};

// Workspace of a prefill: rotated keys per map, query angle tables per map,
// and for half-split pairing the query in adjacent order.
PrefillLayout prefill_layout(int eff_kind, bool half, long long B, long long S, int Hq, int Hkv, int D) {
  PrefillLayout L{};
  L.nmaps = eff_kind == ROPEATTN_NOPE ? 0 : (eff_kind == ROPEATTN_BIFOCAL ? 2 : 1);
  L.half = half;
  L.krot_bytes = align_up(static_cast<size_t>(B) * S * Hkv * D * 2, 256);
  L.tab_bytes = align_up(static_cast<size_t>(S) * (D / 2) * sizeof(float2), 256);
  size_t off = 0;
  for (int i = 0; i < L.nmaps; ++i) { L.off_krot[i] = off; off += L.krot_bytes; }
  for (int i = 0; i < L.nmaps; ++i) { L.off_tab[i] = off; off += L.tab_bytes; }
  L.off_q = off;
  if (half) off += align_up(static_cast<size_t>(B) * S * Hq * D * 2, 256);
  L.total = off;
  return L;
}

template <int D, int NST>
int launch_prefill(const CUtensorMap& tq, const CUtensorMap& tk0, const CUtensorMap& tk1, const CUtensorMap& tv,
                   const PrefillParams& pp, int grid, cudaStream_t st) {
  using L = PrefillSmem<D, NST>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(prefill_kernel<D, NST>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
  });
  if (attr_err != cudaSuccess) return cuda_fail(attr_err, "cudaFuncSetAttribute(prefill)");
  prefill_kernel<D, NST><<<grid, PrefillShape<D>::kThreads, L::kAlloc, st>>>(tq, tk0, tk1, tv, pp);
  CUDA_TRY(cudaGetLastError(), "prefill launch");
  return ROPEATTN_OK;
}

// Query rows per CTA and keys per K/V tile of the prefill kernel (PrefillShape).
int prefill_block_rows(int D) { return D == 256 ? PrefillShape<256>::kBlockRows : PrefillShape<128>::kBlockRows; }
int prefill_bn(int D) { return D == 256 ? PrefillShape<256>::kBN : PrefillShape<128>::kBN; }

// One prefill attention launch for the head dimension.
int launch_prefill_d(int D, const CUtensorMap& tq, const CUtensorMap& tk0, const CUtensorMap& tk1,
                     const CUtensorMap& tv, const PrefillParams& pp, int grid, cudaStream_t st) {
  if (D == 256) return launch_prefill<256, 6>(tq, tk0, tk1, tv, pp, grid, st);
  if (D == 128) return launch_prefill<128, 4>(tq, tk0, tk1, tv, pp, grid, st);
  return launch_prefill<64, 8>(tq, tk0, tk1, tv, pp, grid, st);
}

struct DecodeLayout {
  int nsplit;
  size_t off_q, off_o, off_ml, off_cnt, total;
};

// One CTA per SM is resident (shared-memory ring), so the grid is sized to
// one wave: splits per (batch, kv head) = SMs / (B * Hkv), at least one.
int decode_nsplit(long long B, long long keys, int Hkv) {
  long long want = static_cast<long long>(sm_count()) / (Hkv * B);
  long long cap = (keys + 255) / 256;
  if (cap > kTcMaxSplits) cap = kTcMaxSplits;   // the merge stages every split's (m, l) on chip
  long long ns = want < cap ? want : cap;
  return static_cast<int>(ns < 1 ? 1 : ns);
}

DecodeLayout decode_layout(long long B, long long keys, int Hq, int Hkv, int D) {
  DecodeLayout L{};
  L.nsplit = decode_nsplit(B, keys, Hkv);
  size_t slots = static_cast<size_t>(B) * Hq * L.nsplit;
  L.off_q = 0;   // the query in adjacent order (half-split pairing); kept for either pairing
  L.off_o = align_up(static_cast<size_t>(B) * Hq * D * 2, 256);
  L.off_ml = L.off_o + align_up(slots * D * sizeof(float), 256);
  L.off_cnt = L.off_ml + align_up(slots * sizeof(float2), 256);
  L.total = L.off_cnt + align_up(static_cast<size_t>(B) * Hkv * sizeof(int), 256);
  return L;
}

template <int D, int GP, int ROT>
int launch_decode_tc_rot(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeParams& dp, dim3 grid,
                         cudaStream_t st) {
  using L = DecodeTcShape<D, GP, ROT>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(decode_tc_kernel<D, GP, ROT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    L::kAlloc);
  });
  if (attr_err != cudaSuccess) return cuda_fail(attr_err, "cudaFuncSetAttribute(decode_tc)");
  decode_tc_kernel<D, GP, ROT><<<grid, kTcThreads, L::kAlloc, st>>>(tk, tv, dp);
  CUDA_TRY(cudaGetLastError(), "decode launch");
  return ROPEATTN_OK;
}

// Tensor-core decode (head_dim 64 and 128): the group's query heads padded to
// a power of two GP <= 16; remote keys rotated in shared memory for the
// bifocal map.
template <int D>
int launch_decode_tc(int grp, const CUtensorMap& tk, const CUtensorMap& tv, const DecodeParams& dp, dim3 grid,
                     cudaStream_t st) {
  const bool r = dp.bifocal != 0;
  if (grp <= 2) return r ? launch_decode_tc_rot<D, 2, 1>(tk, tv, dp, grid, st) : launch_decode_tc_rot<D, 2, 0>(tk, tv, dp, grid, st);
  if (grp <= 4) return r ? launch_decode_tc_rot<D, 4, 1>(tk, tv, dp, grid, st) : launch_decode_tc_rot<D, 4, 0>(tk, tv, dp, grid, st);
  if (grp <= 8) return r ? launch_decode_tc_rot<D, 8, 1>(tk, tv, dp, grid, st) : launch_decode_tc_rot<D, 8, 0>(tk, tv, dp, grid, st);
  return r ? launch_decode_tc_rot<D, 16, 1>(tk, tv, dp, grid, st) : launch_decode_tc_rot<D, 16, 0>(tk, tv, dp, grid, st);
}

}  // namespace

extern "C" {

const char* ropeattn_last_error(void) { return g_last_error.c_str(); }

int ropeattn_version(void) { return kVersion; }

int ropeattn_wait_selftest(int64_t limit_ns, int32_t* d_result, void* stream) {
  g_last_error.clear();
  if (limit_ns < 1000 || limit_ns > 1000000000LL)
    return fail(ROPEATTN_ERR_INVALID_ARG, "limit_ns must be in [1e3, 1e9]");
  if (!d_result) return fail(ROPEATTN_ERR_INVALID_ARG, "d_result is NULL");
  int rc = check_device();
  if (rc) return rc;
  wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<unsigned long long>(limit_ns),
                                                                      d_result);
  CUDA_TRY(cudaGetLastError(), "selftest launch");
  return ROPEATTN_OK;
}

int ropeattn_status(void) {
  g_last_error.clear();
  CUDA_TRY(cudaDeviceSynchronize(), "cudaDeviceSynchronize");
  int v = 0, zero = 0;
  CUDA_TRY(cudaMemcpyFromSymbol(&v, ropeattn::g_status, sizeof(int)), "read status");
  CUDA_TRY(cudaMemcpyToSymbol(ropeattn::g_status, &zero, sizeof(int)), "clear status");
  if (v & kStatusTimeout) return fail(ROPEATTN_ERR_TIMEOUT, "a kernel gave up on a bounded wait");
  return ROPEATTN_OK;
}

int ropeattn_posmap(const ropeattn_params* params, int64_t L, int32_t* d_pos_local, int32_t* d_pos_remote,
                    int32_t* h_G, void* stream) {
  g_last_error.clear();
  PosMap m;
  int eff;
  int rc = check_params(params, L, 64, &m, &eff);
  if (rc) return rc;
  if (L > 0 && !d_pos_local) return fail(ROPEATTN_ERR_INVALID_ARG, "d_pos_local is NULL");
  if (L > 0 && params->kind == ROPEATTN_BIFOCAL && !d_pos_remote)
    return fail(ROPEATTN_ERR_INVALID_ARG, "d_pos_remote is required for BIFOCAL");
  if (h_G) *h_G = m.G;
  if (L == 0) return ROPEATTN_OK;
  const int threads = 256;
  const long long blocks = (L + threads - 1) / threads;
  posmap_kernel<<<static_cast<unsigned>(blocks), threads, 0, static_cast<cudaStream_t>(stream)>>>(
      m, static_cast<int>(L), d_pos_local, d_pos_remote);
  CUDA_TRY(cudaGetLastError(), "posmap launch");
  return ROPEATTN_OK;
}

int ropeattn_cache_write(const void* k, const void* v, void* k_cache, void* v_cache, int64_t B, int64_t start,
                         int64_t count, int64_t cache_len, int32_t Hkv, int32_t D, const ropeattn_params* params,
                         void* stream) {
  g_last_error.clear();
  if (B < 0 || start < 0 || count < 0 || cache_len < 0)
    return fail(ROPEATTN_ERR_INVALID_ARG, "B, start, count and cache_len must be >= 0");
  if (start + count > cache_len)
    return fail(ROPEATTN_ERR_INVALID_ARG, "start + count (%lld) exceeds cache_len (%lld)",
                static_cast<long long>(start + count), static_cast<long long>(cache_len));
  int rc = check_shapes(B, cache_len, Hkv, Hkv, D);
  if (rc) return rc;
  PosMap m;
  int eff;
  rc = check_params(params, cache_len, D, &m, &eff);
  if (rc) return rc;
  if (B == 0 || count == 0) return ROPEATTN_OK;
  if (!k || !k_cache) return fail(ROPEATTN_ERR_INVALID_ARG, "k and k_cache must not be NULL");
  if ((v == nullptr) != (v_cache == nullptr))
    return fail(ROPEATTN_ERR_INVALID_ARG, "v and v_cache must be both given or both NULL");
  if ((reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(k_cache) | reinterpret_cast<uintptr_t>(v) |
       reinterpret_cast<uintptr_t>(v_cache)) & 15u)
    return fail(ROPEATTN_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  rc = check_device();
  if (rc) return rc;
  CacheArgs a{};
  a.k = static_cast<const uint32_t*>(k);
  a.v = static_cast<const uint32_t*>(v);
  a.k_cache = static_cast<uint32_t*>(k_cache);
  a.v_cache = static_cast<uint32_t*>(v_cache);
  a.start = start;
  a.count = count;
  a.cache_len = cache_len;
  a.B = static_cast<int>(B);
  a.Hkv = Hkv;
  a.D = D;
  a.half = half_pairing(params) ? 1 : 0;
  m.kind = params->kind == ROPEATTN_BIFOCAL ? ROPEATTN_STANDARD : params->kind;  // primary position: t
  a.m = m;
  fill_theta(params, D, a.theta);
  const int rows = 256 / (D / 8);   // four rotation pairs per thread
  cache_write_kernel<<<static_cast<unsigned>((count + rows - 1) / rows), 256, 0, static_cast<cudaStream_t>(stream)>>>(a);
  CUDA_TRY(cudaGetLastError(), "cache_write launch");
  return ROPEATTN_OK;
}

size_t ropeattn_prefill_workspace_size(const ropeattn_params* params, int64_t B, int64_t S, int32_t Hq,
                                       int32_t Hkv, int32_t D) {
  PosMap m;
  int eff;
  if (check_params(params, S, D, &m, &eff) || check_shapes(B, S, Hq, Hkv, D)) return 0;
  return prefill_layout(eff, half_pairing(params), B, S, Hq, Hkv, D).total;
}

}  // extern "C"

namespace {

enum : int { kStagePrepare = 1, kStageAttend = 2 };

int prefill_impl(int stages, const void* q, const void* k, const void* v, float* out, float* lse, int64_t B,
                 int64_t S, int32_t Hq, int32_t Hkv, int32_t D, const ropeattn_params* params, void* workspace,
                 size_t workspace_bytes, void* stream) {
  g_last_error.clear();
  int rc = check_shapes(B, S, Hq, Hkv, D);
  if (rc) return rc;
  PosMap m;
  int eff;
  rc = check_params(params, S, D, &m, &eff);
  if (rc) return rc;
  if (B == 0 || S == 0) return ROPEATTN_OK;
  if (!k) return fail(ROPEATTN_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(k)) return fail(ROPEATTN_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  if (stages & kStageAttend) {
    if (!q || !v || !out || !lse) return fail(ROPEATTN_ERR_INVALID_ARG, "null tensor pointer");
    if (!aligned16(q) || !aligned16(v) || !aligned16(out) || !aligned16(lse))
      return fail(ROPEATTN_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  }
  if ((static_cast<long long>((S + prefill_block_rows(D) - 1) / prefill_block_rows(D))) * Hq * B > 0x7fffffffLL)
    return fail(ROPEATTN_ERR_INVALID_ARG, "too many query tiles");
  rc = check_device();
  if (rc) return rc;
  const PrefillLayout lay = prefill_layout(eff, half_pairing(params), B, S, Hq, Hkv, D);
  if (lay.total > 0) {
    if (!workspace || workspace_bytes < lay.total)
      return fail(ROPEATTN_ERR_WORKSPACE, "workspace of %zu bytes needed (got %zu)", lay.total,
                  workspace ? workspace_bytes : size_t(0));
    if (reinterpret_cast<uintptr_t>(workspace) & 255u)
      return fail(ROPEATTN_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  m.kind = eff;

  // workspace views: keys rotated once per map, and the query angle tables
  const void* kmap0 = k;
  const void* kmap1 = k;
  PrefillParams pp{};
  if (lay.nmaps > 0) {
    PrepArgs a{};
    a.k = static_cast<const uint32_t*>(k);
    a.k_rot0 = reinterpret_cast<uint32_t*>(ws + lay.off_krot[0]);
    a.k_rot1 = lay.nmaps > 1 ? reinterpret_cast<uint32_t*>(ws + lay.off_krot[1]) : nullptr;
    a.tab0 = reinterpret_cast<float2*>(ws + lay.off_tab[0]);
    a.tab1 = lay.nmaps > 1 ? reinterpret_cast<float2*>(ws + lay.off_tab[1]) : nullptr;
    a.B = static_cast<int>(B);
    a.S = static_cast<int>(S);
    a.Hkv = Hkv;
    a.D = D;
    a.half = lay.half ? 1 : 0;
    a.m = m;
    if (stages & kStagePrepare) {
      fill_theta(params, D, a.theta);
      const int rows = 256 / (D / 8);   // four rotation pairs per thread
      rope_prep_kernel<<<static_cast<unsigned>((S + rows - 1) / rows), 256, 0, st>>>(a);
      CUDA_TRY(cudaGetLastError(), "rope_prep launch");
    }
    kmap0 = a.k_rot0;
    kmap1 = lay.nmaps > 1 ? static_cast<const void*>(a.k_rot1) : kmap0;
    pp.tab0 = a.tab0;
    pp.tab1 = a.tab1;
  }
  if (!(stages & kStageAttend)) return ROPEATTN_OK;
  if (lay.half) {
    if ((rc = launch_interleave(q, ws + lay.off_q, B * S * Hq, D, st))) return rc;
    q = ws + lay.off_q;
  }

  CUtensorMap tq, tk0, tk1, tv;
  if ((rc = make_map(&tq, q, D, Hq, S, B, 64, kBM, true))) return rc;
  if ((rc = make_map(&tk0, kmap0, D, Hkv, S, B, 64, prefill_bn(D), true))) return rc;
  if ((rc = make_map(&tk1, kmap1, D, Hkv, S, B, 64, prefill_bn(D), true))) return rc;
  if ((rc = make_map(&tv, v, D, Hkv, S, B, 64, prefill_bn(D), true))) return rc;
  pp.out = out;
  pp.lse = lse;
  pp.B = static_cast<int>(B);
  pp.S = static_cast<int>(S);
  pp.Sk = static_cast<int>(S);
  pp.q_off = 0;
  pp.Hq = Hq;
  pp.Hkv = Hkv;
  pp.nqb = static_cast<int>((S + prefill_block_rows(D) - 1) / prefill_block_rows(D));
  pp.kind = eff;
  pp.window = m.window;
  pp.w0 = m.w0;
  pp.scale_log2 = scale_log2(params, D);
  const int grid = pp.nqb * Hq * static_cast<int>(B);
  return launch_prefill_d(D, tq, tk0, tk1, tv, pp, grid, st);
}

struct ChunkLayout {
  size_t off_krem, off_tab0, off_tab1, off_q, total;
  bool remote, tables, half;
};

ChunkLayout chunk_layout(int eff_kind, bool half, long long B, long long L, long long count, int Hq, int Hkv, int D) {
  ChunkLayout c{};
  c.remote = eff_kind == ROPEATTN_BIFOCAL;
  c.tables = eff_kind != ROPEATTN_NOPE;
  c.half = half;
  size_t off = 0;
  c.off_krem = off;
  if (c.remote) off += align_up(static_cast<size_t>(B) * L * Hkv * D * 2, 256);
  const size_t tab = align_up(static_cast<size_t>(count) * (D / 2) * sizeof(float2), 256);
  c.off_tab0 = off;
  if (c.tables) off += tab;
  c.off_tab1 = off;
  if (c.remote) off += tab;
  c.off_q = off;
  if (half) off += align_up(static_cast<size_t>(B) * count * Hq * D * 2, 256);
  c.total = off;
  return c;
}

}  // namespace

extern "C" {

size_t ropeattn_prefill_chunk_workspace_size(const ropeattn_params* params, int64_t B, int64_t start, int64_t count,
                                             int32_t Hq, int32_t Hkv, int32_t D) {
  PosMap m;
  int eff;
  if (start < 0 || count < 0 || check_params(params, start + count, D, &m, &eff) ||
      check_shapes(B, start + count, Hq, Hkv, D))
    return 0;
  return chunk_layout(eff, half_pairing(params), B, start + count, count, Hq, Hkv, D).total;
}

int ropeattn_prefill_chunk(const void* q, const void* k_cache, const void* v_cache, float* out, float* lse,
                           int64_t B, int64_t start, int64_t count, int32_t Hq, int32_t Hkv, int32_t D,
                           const ropeattn_params* params, void* workspace, size_t workspace_bytes, void* stream) {
  return ropeattn_prefill_chunk_cache(q, k_cache, v_cache, out, lse, B, start, count, start + count, Hq, Hkv, D,
                                      params, workspace, workspace_bytes, stream);
}

int ropeattn_prefill_chunk_cache(const void* q, const void* k_cache, const void* v_cache, float* out, float* lse,
                                 int64_t B, int64_t start, int64_t count, int64_t cache_len, int32_t Hq, int32_t Hkv,
                                 int32_t D, const ropeattn_params* params, void* workspace, size_t workspace_bytes,
                                 void* stream) {
  g_last_error.clear();
  if (start < 0 || count < 0) return fail(ROPEATTN_ERR_INVALID_ARG, "start and count must be >= 0");
  const long long L = start + count;
  if (cache_len < L || cache_len > kMaxPos)
    return fail(ROPEATTN_ERR_INVALID_ARG, "cache_len (%lld) must be in [start + count, 2^31)",
                static_cast<long long>(cache_len));
  int rc = check_shapes(B, L, Hq, Hkv, D);
  if (rc) return rc;
  PosMap m;
  int eff;
  rc = check_params(params, L, D, &m, &eff);
  if (rc) return rc;
  if (B == 0 || count == 0) return ROPEATTN_OK;
  if (!q || !k_cache || !v_cache || !out || !lse) return fail(ROPEATTN_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) || !aligned16(lse))
    return fail(ROPEATTN_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  if ((static_cast<long long>((count + prefill_block_rows(D) - 1) / prefill_block_rows(D))) * Hq * B > 0x7fffffffLL)
    return fail(ROPEATTN_ERR_INVALID_ARG, "too many query tiles");
  rc = check_device();
  if (rc) return rc;
  const ChunkLayout lay = chunk_layout(eff, half_pairing(params), B, L, count, Hq, Hkv, D);
  if (lay.total > 0) {
    if (!workspace || workspace_bytes < lay.total)
      return fail(ROPEATTN_ERR_WORKSPACE, "workspace of %zu bytes needed (got %zu)", lay.total,
                  workspace ? workspace_bytes : size_t(0));
    if (reinterpret_cast<uintptr_t>(workspace) & 255u)
      return fail(ROPEATTN_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  m.kind = eff;

  PrefillParams pp{};
  const void* kmap1 = k_cache;
  if (lay.tables) {
    ChunkPrepArgs a{};
    a.k_cache = static_cast<const uint32_t*>(k_cache);
    a.k_rem = lay.remote ? reinterpret_cast<uint32_t*>(ws + lay.off_krem) : nullptr;
    a.tab0 = reinterpret_cast<float2*>(ws + lay.off_tab0);
    a.tab1 = lay.remote ? reinterpret_cast<float2*>(ws + lay.off_tab1) : nullptr;
    a.B = static_cast<int>(B);
    a.L = static_cast<int>(L);
    a.cache_rows = cache_len;
    a.Hkv = Hkv;
    a.D = D;
    a.start = static_cast<int>(start);
    a.m = m;
    fill_theta(params, D, a.theta);
    const int rows = 256 / (D / 8);   // four rotation pairs per thread
    chunk_prep_kernel<<<static_cast<unsigned>((L + rows - 1) / rows), 256, 0, st>>>(a);
    CUDA_TRY(cudaGetLastError(), "chunk_prep launch");
    pp.tab0 = a.tab0;
    pp.tab1 = a.tab1;
    if (lay.remote) kmap1 = a.k_rem;
  }
  if (lay.half) {
    if ((rc = launch_interleave(q, ws + lay.off_q, B * count * Hq, D, st))) return rc;
    q = ws + lay.off_q;
  }
  CUtensorMap tq, tk0, tk1, tv;
  if ((rc = make_map(&tq, q, D, Hq, count, B, 64, kBM, true))) return rc;
  if ((rc = make_map(&tk0, k_cache, D, Hkv, L, B, 64, prefill_bn(D), true, cache_len))) return rc;
  if ((rc = make_map(&tk1, kmap1, D, Hkv, L, B, 64, prefill_bn(D), true, lay.remote ? 0 : cache_len))) return rc;
  if ((rc = make_map(&tv, v_cache, D, Hkv, L, B, 64, prefill_bn(D), true, cache_len))) return rc;
  pp.out = out;
  pp.lse = lse;
  pp.B = static_cast<int>(B);
  pp.S = static_cast<int>(count);
  pp.Sk = static_cast<int>(L);
  pp.q_off = static_cast<int>(start);
  pp.Hq = Hq;
  pp.Hkv = Hkv;
  pp.nqb = static_cast<int>((count + prefill_block_rows(D) - 1) / prefill_block_rows(D));
  pp.kind = eff;
  pp.window = m.window;
  pp.w0 = m.w0;
  pp.scale_log2 = scale_log2(params, D);
  const int grid = pp.nqb * Hq * static_cast<int>(B);
  return launch_prefill_d(D, tq, tk0, tk1, tv, pp, grid, st);
}

size_t ropeattn_prefill_three_call_workspace_size(const ropeattn_params* params, int64_t B, int64_t S, int32_t Hq,
                                                  int32_t Hkv, int32_t D) {
  PosMap m;
  int eff;
  if (check_params(params, S, D, &m, &eff) || check_shapes(B, S, Hq, Hkv, D) || eff != ROPEATTN_BIFOCAL) return 0;
  const size_t o = align_up(static_cast<size_t>(B) * S * Hq * D * sizeof(float), 256);
  const size_t l = align_up(static_cast<size_t>(B) * Hq * S * sizeof(float), 256);
  return prefill_layout(eff, half_pairing(params), B, S, Hq, Hkv, D).total + 2 * o + 2 * l;
}

int ropeattn_prefill_three_call(const void* q, const void* k, const void* v, float* out, float* lse, int64_t B,
                                int64_t S, int32_t Hq, int32_t Hkv, int32_t D, const ropeattn_params* params,
                                void* workspace, size_t workspace_bytes, void* stream) {
  g_last_error.clear();
  int rc = check_shapes(B, S, Hq, Hkv, D);
  if (rc) return rc;
  PosMap m;
  int eff;
  rc = check_params(params, S, D, &m, &eff);
  if (rc) return rc;
  if (eff != ROPEATTN_BIFOCAL)
    return fail(ROPEATTN_ERR_INVALID_ARG, "the three-call prefill needs a bifocal map with G > 1 and w0 < S-1");
  if (B == 0 || S == 0) return ROPEATTN_OK;
  if (!q || !k || !v || !out || !lse) return fail(ROPEATTN_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse))
    return fail(ROPEATTN_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  if ((static_cast<long long>((S + prefill_block_rows(D) - 1) / prefill_block_rows(D))) * Hq * B > 0x7fffffffLL)
    return fail(ROPEATTN_ERR_INVALID_ARG, "too many query tiles");
  rc = check_device();
  if (rc) return rc;
  const PrefillLayout lay = prefill_layout(eff, half_pairing(params), B, S, Hq, Hkv, D);
  const size_t obytes = align_up(static_cast<size_t>(B) * S * Hq * D * sizeof(float), 256);
  const size_t lbytes = align_up(static_cast<size_t>(B) * Hq * S * sizeof(float), 256);
  const size_t need = lay.total + 2 * obytes + 2 * lbytes;
  if (!workspace || workspace_bytes < need)
    return fail(ROPEATTN_ERR_WORKSPACE, "workspace of %zu bytes needed (got %zu)", need,
                workspace ? workspace_bytes : size_t(0));
  if (reinterpret_cast<uintptr_t>(workspace) & 255u)
    return fail(ROPEATTN_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  m.kind = eff;
  float* oA = reinterpret_cast<float*>(ws + lay.total);
  float* oC = reinterpret_cast<float*>(ws + lay.total + obytes);
  float* lA = reinterpret_cast<float*>(ws + lay.total + 2 * obytes);
  float* lC = reinterpret_cast<float*>(ws + lay.total + 2 * obytes + lbytes);

  // keys rotated to both maps and the query angle tables, as in the fused prefill
  PrepArgs a{};
  a.k = static_cast<const uint32_t*>(k);
  a.k_rot0 = reinterpret_cast<uint32_t*>(ws + lay.off_krot[0]);
  a.k_rot1 = reinterpret_cast<uint32_t*>(ws + lay.off_krot[1]);
  a.tab0 = reinterpret_cast<float2*>(ws + lay.off_tab[0]);
  a.tab1 = reinterpret_cast<float2*>(ws + lay.off_tab[1]);
  a.B = static_cast<int>(B);
  a.S = static_cast<int>(S);
  a.Hkv = Hkv;
  a.D = D;
  a.half = lay.half ? 1 : 0;
  a.m = m;
  fill_theta(params, D, a.theta);
  const int prow = 256 / (D / 8);   // four rotation pairs per thread
  rope_prep_kernel<<<static_cast<unsigned>((S + prow - 1) / prow), 256, 0, st>>>(a);
  CUDA_TRY(cudaGetLastError(), "rope_prep launch");
  if (lay.half) {
    if ((rc = launch_interleave(q, ws + lay.off_q, B * S * Hq, D, st))) return rc;
    q = ws + lay.off_q;
  }

  CUtensorMap tq, tk0, tk1, tv;
  if ((rc = make_map(&tq, q, D, Hq, S, B, 64, kBM, true))) return rc;
  if ((rc = make_map(&tk0, a.k_rot0, D, Hkv, S, B, 64, prefill_bn(D), true))) return rc;
  if ((rc = make_map(&tk1, a.k_rot1, D, Hkv, S, B, 64, prefill_bn(D), true))) return rc;
  if ((rc = make_map(&tv, v, D, Hkv, S, B, 64, prefill_bn(D), true))) return rc;
  PrefillParams pp{};
  pp.tab0 = a.tab0;
  pp.tab1 = a.tab1;
  pp.B = static_cast<int>(B);
  pp.S = static_cast<int>(S);
  pp.Sk = static_cast<int>(S);
  pp.q_off = 0;
  pp.Hq = Hq;
  pp.Hkv = Hkv;
  pp.nqb = static_cast<int>((S + prefill_block_rows(D) - 1) / prefill_block_rows(D));
  pp.kind = ROPEATTN_STANDARD;   // each call writes its own normalised output and LSE
  pp.window = m.window;
  pp.w0 = m.w0;
  pp.scale_log2 = scale_log2(params, D);
  pp.forced = 1;
  const int grid = pp.nqb * Hq * static_cast<int>(B);
  // (A) sliding window w0, exact positions; (B) full causal, remote positions;
  // (C) sliding window w0, remote positions (Jet-Long §3.3)
  const int calls[3][3] = {{m.w0, 0, 0}, {kInf, 0, 1}, {m.w0, 0, 1}};
  float* outs[3] = {oA, out, oC};
  float* lses[3] = {lA, lse, lC};
  for (int c = 0; c < 3; ++c) {
    pp.forced_lo = calls[c][0];
    pp.forced_hi = calls[c][1];
    pp.forced_sel = calls[c][2];
    pp.out = outs[c];
    pp.lse = lses[c];
    rc = launch_prefill_d(D, tq, tk0, tk1, tv, pp, grid, st);
    if (rc) return rc;
  }
  MergeArgs ma{};
  ma.oA = oA;
  ma.oC = oC;
  ma.out = out;
  ma.lA = lA;
  ma.lC = lC;
  ma.lse = lse;
  ma.rows = static_cast<long long>(B) * S * Hq;
  ma.S = static_cast<int>(S);
  ma.Hq = Hq;
  ma.D = D;
  three_call_merge_kernel<<<static_cast<unsigned>((ma.rows * 32 + 255) / 256), 256, 0, st>>>(ma);
  CUDA_TRY(cudaGetLastError(), "merge launch");
  return ROPEATTN_OK;
}

int ropeattn_prefill(const void* q, const void* k, const void* v, float* out, float* lse, int64_t B, int64_t S,
                     int32_t Hq, int32_t Hkv, int32_t D, const ropeattn_params* params, void* workspace,
                     size_t workspace_bytes, void* stream) {
  return prefill_impl(kStagePrepare | kStageAttend, q, k, v, out, lse, B, S, Hq, Hkv, D, params, workspace,
                      workspace_bytes, stream);
}

int ropeattn_prefill_prepare(const void* k, int64_t B, int64_t S, int32_t Hq, int32_t Hkv, int32_t D,
                             const ropeattn_params* params, void* workspace, size_t workspace_bytes, void* stream) {
  return prefill_impl(kStagePrepare, nullptr, k, nullptr, nullptr, nullptr, B, S, Hq, Hkv, D, params, workspace,
                      workspace_bytes, stream);
}

int ropeattn_prefill_attend(const void* q, const void* k, const void* v, float* out, float* lse, int64_t B,
                            int64_t S, int32_t Hq, int32_t Hkv, int32_t D, const ropeattn_params* params,
                            void* workspace, size_t workspace_bytes, void* stream) {
  return prefill_impl(kStageAttend, q, k, v, out, lse, B, S, Hq, Hkv, D, params, workspace, workspace_bytes,
                      stream);
}

size_t ropeattn_decode_workspace_size(int64_t B, int64_t n, int32_t Hq, int32_t Hkv, int32_t D) {
  if (check_shapes(B, n, Hq, Hkv, D) || B == 0 || n == 0) return 0;
  return decode_layout(B, n, Hq, Hkv, D).total;
}

int ropeattn_decode(const void* q, const void* k_cache, const void* v_cache, float* out, float* lse, int64_t B,
                    int64_t n, int32_t Hq, int32_t Hkv, int32_t D, const ropeattn_params* params, void* workspace,
                    size_t workspace_bytes, void* stream) {
  return ropeattn_decode_cache(q, k_cache, v_cache, out, lse, B, n, n, Hq, Hkv, D, params, workspace, workspace_bytes,
                               stream);
}

int ropeattn_decode_cache(const void* q, const void* k_cache, const void* v_cache, float* out, float* lse, int64_t B,
                          int64_t n, int64_t cache_len, int32_t Hq, int32_t Hkv, int32_t D,
                          const ropeattn_params* params, void* workspace, size_t workspace_bytes, void* stream) {
  g_last_error.clear();
  int rc = check_shapes(B, n, Hq, Hkv, D);
  if (rc) return rc;
  if (cache_len < n || cache_len > kMaxPos)
    return fail(ROPEATTN_ERR_INVALID_ARG, "cache_len (%lld) must be in [n, 2^31)", static_cast<long long>(cache_len));
  PosMap m;
  int eff;
  rc = check_params(params, n, D, &m, &eff);
  if (rc) return rc;
  if (B == 0 || n == 0) return ROPEATTN_OK;
  const int grp = Hq / Hkv;
  if (grp > 16) return fail(ROPEATTN_ERR_INVALID_ARG, "decode supports Hq/Hkv <= 16");
  if (!q || !k_cache || !v_cache || !out || !lse) return fail(ROPEATTN_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) || !aligned16(lse))
    return fail(ROPEATTN_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  rc = check_device();
  if (rc) return rc;
  const long long t = n - 1;
  const long long k_begin = eff == ROPEATTN_PERIODIC ? (n > m.window ? n - m.window : 0) : 0;
  const long long keys = n - k_begin;
  const DecodeLayout lay = decode_layout(B, keys, Hq, Hkv, D);
  const size_t need = ropeattn_decode_workspace_size(B, n, Hq, Hkv, D);
  if (!workspace || workspace_bytes < need)
    return fail(ROPEATTN_ERR_WORKSPACE, "workspace of %zu bytes needed (got %zu)", need,
                workspace ? workspace_bytes : size_t(0));
  if (reinterpret_cast<uintptr_t>(workspace) & 255u)
    return fail(ROPEATTN_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);

  if (half_pairing(params)) {
    if ((rc = launch_interleave(q, ws + lay.off_q, B * Hq, D, st))) return rc;
    q = ws + lay.off_q;
  }
  DecodeParams dp{};
  dp.q = static_cast<const __nv_bfloat16*>(q);
  dp.out = out;
  dp.lse = lse;
  dp.part_o = reinterpret_cast<float*>(ws + lay.off_o);
  dp.part_ml = reinterpret_cast<float2*>(ws + lay.off_ml);
  dp.counters = reinterpret_cast<int*>(ws + lay.off_cnt);
  dp.B = static_cast<int>(B);
  dp.n = static_cast<int>(n);
  dp.Hq = Hq;
  dp.Hkv = Hkv;
  dp.nsplit = lay.nsplit;
  dp.keys_per_split = static_cast<int>(align_up(static_cast<size_t>((keys + lay.nsplit - 1) / lay.nsplit), kTcKeys));
  dp.k_begin = static_cast<int>(k_begin);
  dp.bifocal = eff == ROPEATTN_BIFOCAL ? 1 : 0;
  dp.k_local = dp.bifocal ? static_cast<int>(t - m.w0 > 0 ? t - m.w0 : 0) : 0;
  m.kind = eff;
  dp.m = m;
  dp.scale_log2 = scale_log2(params, D);
  fill_turns(params, D, dp.turns);

  // 64-column blocks with the 128-byte swizzle (tcgen05 operands): K in
  // 128-key tiles, V in 64-key halves
  CUtensorMap tk, tv;
  if ((rc = make_map(&tk, k_cache, D, Hkv, n, B, 64, kTcKeys, true, cache_len))) return rc;
  if ((rc = make_map(&tv, v_cache, D, Hkv, n, B, 64, kTcKeys / 2, true, cache_len))) return rc;
  CUDA_TRY(cudaMemsetAsync(dp.counters, 0, static_cast<size_t>(B) * Hkv * sizeof(int), st), "memset counters");
  dim3 grid(lay.nsplit, Hkv, static_cast<unsigned>(B));
  if (D == 256) return launch_decode_tc<256>(grp, tk, tv, dp, grid, st);
  if (D == 128) return launch_decode_tc<128>(grp, tk, tv, dp, grid, st);
  return launch_decode_tc<64>(grp, tk, tv, dp, grid, st);
}


}  // extern "C"

// ---------------------------------------------------------------------------
// Decode without a caller-provided workspace: the scratch is a fixed array
// owned by the library. Callers that cannot allocate device memory pass only
// inputs and outputs.
// ---------------------------------------------------------------------------
static constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

// Device address of g_noalloc_scratch on the current device (the host-side
// name is only a stand-in, never a device address). Looked up on every call:
// it is a table lookup that allocates nothing, and a cached address would
// outlive a device reset that reloads the library's device code.
int noalloc_scratch_ptr(void** out) {
  void* p = nullptr;
  CUDA_TRY(cudaGetSymbolAddress(&p, g_noalloc_scratch), "cudaGetSymbolAddress(scratch)");
  *out = p;
  return ROPEATTN_OK;
}

}  // namespace

extern "C" size_t ropeattn_decode_unfused_workspace_size(int64_t B, int64_t n, int32_t Hq, int32_t Hkv, int32_t D) {
  if (check_shapes(B, n, Hq, Hkv, D) || B == 0 || n == 0) return 0;
  return align_up(static_cast<size_t>(B) * n * Hkv * D * 2, 256) + decode_layout(B, n, Hq, Hkv, D).total;
}

int ropeattn_decode_unfused(const void* q, const void* k_cache, const void* v_cache, float* out, float* lse,
                            int64_t B, int64_t n, int32_t Hq, int32_t Hkv, int32_t D, const ropeattn_params* params,
                            void* workspace, size_t workspace_bytes, void* stream) {
  g_last_error.clear();
  int rc = check_shapes(B, n, Hq, Hkv, D);
  if (rc) return rc;
  PosMap m;
  int eff;
  rc = check_params(params, n, D, &m, &eff);
  if (rc) return rc;
  if (eff != ROPEATTN_BIFOCAL)
    return fail(ROPEATTN_ERR_INVALID_ARG, "the unfused decode needs a bifocal map with G > 1 and w0 < n-1");
  if (B == 0 || n == 0) return ROPEATTN_OK;
  if (!q || !k_cache || !v_cache || !out || !lse) return fail(ROPEATTN_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(k_cache)) return fail(ROPEATTN_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  const size_t kbytes = align_up(static_cast<size_t>(B) * n * Hkv * D * 2, 256);
  const size_t need = kbytes + decode_layout(B, n, Hq, Hkv, D).total;
  if (!workspace || workspace_bytes < need)
    return fail(ROPEATTN_ERR_WORKSPACE, "workspace of %zu bytes needed (got %zu)", need,
                workspace ? workspace_bytes : size_t(0));
  if (reinterpret_cast<uintptr_t>(workspace) & 255u)
    return fail(ROPEATTN_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  rc = check_device();
  if (rc) return rc;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const long long t = n - 1;
  UnfusedRotArgs a{};
  a.k_cache = static_cast<const uint32_t*>(k_cache);
  a.k_out = reinterpret_cast<uint32_t*>(ws);
  a.B = static_cast<int>(B);
  a.n = static_cast<int>(n);
  a.Hkv = Hkv;
  a.D = D;
  a.k_local = static_cast<int>(t - m.w0 > 0 ? t - m.w0 : 0);
  m.kind = eff;
  a.m = m;
  a.dq = pos_remote(m, static_cast<int>(t)) - static_cast<int>(t);
  fill_theta(params, D, a.theta);
  const int rows = 256 / (D / 8);   // four rotation pairs per thread
  unfused_rotate_kernel<<<static_cast<unsigned>((n + rows - 1) / rows), 256, 0, static_cast<cudaStream_t>(stream)>>>(a);
  CUDA_TRY(cudaGetLastError(), "unfused rotate launch");
  // standard RoPE decode over the rotated copy: query at p(t) = t, keys as stored
  ropeattn_params sp = *params;
  sp.kind = ROPEATTN_STANDARD;
  sp.fixed_group = 0;
  return ropeattn_decode(q, ws, v_cache, out, lse, B, n, Hq, Hkv, D, &sp, ws + kbytes, workspace_bytes - kbytes, stream);
}

int ropeattn_decode_noalloc(const void* q, const void* k_cache, const void* v_cache, float* out,
                                       float* lse, int64_t B, int64_t n, int32_t Hq, int32_t Hkv, int32_t D,
                                       const ropeattn_params* params, void* stream) {
  g_last_error.clear();
  const size_t need = ropeattn_decode_workspace_size(B, n, Hq, Hkv, D);
  if (need > kNoAllocScratchBytes)
    return fail(ROPEATTN_ERR_WORKSPACE,
                "this decode needs %zu bytes of scratch; the built-in scratch holds %zu (use ropeattn_decode)", need,
                kNoAllocScratchBytes);
  void* ws = nullptr;
  if (need > 0) {
    const int rc = noalloc_scratch_ptr(&ws);
    if (rc) return rc;
  }
  return ropeattn_decode(q, k_cache, v_cache, out, lse, B, n, Hq, Hkv, D, params, ws, kNoAllocScratchBytes, stream);
}

// ---------------------------------------------------------------------------
// Backward of the prefill
// ---------------------------------------------------------------------------
namespace {

struct BwdLayout {
  int nmaps;
  int Sp;
  size_t off_q[2], off_k[2], off_tab[2], off_lse2, off_delta, total;
};

// Workspace of a backward: per map the rotated queries and keys (bf16) and
// the (cos, sin) table; the log-sum-exp in log2 units and Delta, rows padded
// to a multiple of 64.
BwdLayout bwd_layout(int eff_kind, long long B, long long S, int Hq, int Hkv, int D) {
  BwdLayout L{};
  L.nmaps = eff_kind == ROPEATTN_NOPE ? 0 : (eff_kind == ROPEATTN_BIFOCAL ? 2 : 1);
  L.Sp = static_cast<int>((S + kBwdN - 1) / kBwdN * kBwdN);
  size_t off = 0;
  for (int i = 0; i < L.nmaps; ++i) {
    L.off_q[i] = off;
    off += align_up(static_cast<size_t>(B) * S * Hq * D * 2, 256);
  }
  for (int i = 0; i < L.nmaps; ++i) {
    L.off_k[i] = off;
    off += align_up(static_cast<size_t>(B) * S * Hkv * D * 2, 256);
  }
  for (int i = 0; i < L.nmaps; ++i) {
    L.off_tab[i] = off;
    off += align_up(static_cast<size_t>(S) * (D / 2) * sizeof(float2), 256);
  }
  L.off_lse2 = off;
  off += align_up(static_cast<size_t>(B) * Hq * L.Sp * sizeof(float), 256);
  L.off_delta = off;
  off += align_up(static_cast<size_t>(B) * Hq * L.Sp * sizeof(float), 256);
  L.total = off;
  return L;
}

template <int D>
int launch_backward(const CUtensorMap* ka, const CUtensorMap* kb, const BwdParams& bp, int grid_a, int grid_b,
                    cudaStream_t st) {
  using LA = BwdKVSmem<D>;
  using LB = BwdQSmem<D>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(bwd_dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, LA::kAlloc);
    if (attr_err == cudaSuccess)
      attr_err = cudaFuncSetAttribute(bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, LB::kAlloc);
  });
  if (attr_err != cudaSuccess) return cuda_fail(attr_err, "cudaFuncSetAttribute(backward)");
  bwd_dkdv_kernel<D><<<grid_a, kBwdThreads, LA::kAlloc, st>>>(ka[0], ka[1], ka[2], ka[3], ka[4], ka[5], bp);
  CUDA_TRY(cudaGetLastError(), "backward dK/dV launch");
  bwd_dq_kernel<D><<<grid_b, kBwdThreads, LB::kAlloc, st>>>(kb[0], kb[1], kb[2], kb[3], kb[4], kb[5], bp);
  CUDA_TRY(cudaGetLastError(), "backward dQ launch");
  return ROPEATTN_OK;
}

}  // namespace

extern "C" size_t ropeattn_prefill_backward_workspace_size(const ropeattn_params* params, int64_t B, int64_t S,
                                                           int32_t Hq, int32_t Hkv, int32_t D) {
  PosMap m;
  int eff;
  if (check_shapes(B, S, Hq, Hkv, D) || (D != 64 && D != 128) || check_params(params, S, D, &m, &eff) || B == 0 ||
      S == 0)
    return 0;
  return bwd_layout(eff, B, S, Hq, Hkv, D).total;
}

extern "C" int ropeattn_prefill_backward(const void* q, const void* k, const void* v, const float* out,
                                         const float* lse, const void* dout, float* dq, float* dk, float* dv,
                                         int64_t B, int64_t S, int32_t Hq, int32_t Hkv, int32_t D,
                                         const ropeattn_params* params, void* workspace, size_t workspace_bytes,
                                         void* stream) {
  g_last_error.clear();
  int rc = check_shapes(B, S, Hq, Hkv, D);
  if (rc) return rc;
  if (D != 64 && D != 128) return fail(ROPEATTN_ERR_INVALID_ARG, "the backward supports D = 64 and 128 (got %d)", D);
  PosMap m;
  int eff;
  rc = check_params(params, S, D, &m, &eff);
  if (rc) return rc;
  if (B == 0 || S == 0) return ROPEATTN_OK;
  const void* ptrs[] = {q, k, v, out, lse, dout, dq, dk, dv};
  for (const void* x : ptrs) {
    if (!x) return fail(ROPEATTN_ERR_INVALID_ARG, "null tensor pointer");
    if (!aligned16(x)) return fail(ROPEATTN_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  }
  const long long nkt = (S + kBM - 1) / kBM;
  if (nkt * Hq * B > 0x7fffffffLL) return fail(ROPEATTN_ERR_INVALID_ARG, "too many tiles");
  rc = check_device();
  if (rc) return rc;
  const BwdLayout lay = bwd_layout(eff, B, S, Hq, Hkv, D);
  if (!workspace || workspace_bytes < lay.total)
    return fail(ROPEATTN_ERR_WORKSPACE, "workspace of %zu bytes needed (got %zu)", lay.total,
                workspace ? workspace_bytes : size_t(0));
  if (reinterpret_cast<uintptr_t>(workspace) & 255u)
    return fail(ROPEATTN_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  m.kind = eff;

  // rotated queries and keys per map (the forward's streaming pre-rotation,
  // run over the query rows too), and the angle tables of every position
  const void* qm[2] = {q, q};
  const void* km[2] = {k, k};
  BwdParams bp{};
  if (lay.nmaps > 0) {
    PrepArgs a{};
    a.tab0 = reinterpret_cast<float2*>(ws + lay.off_tab[0]);
    a.tab1 = lay.nmaps > 1 ? reinterpret_cast<float2*>(ws + lay.off_tab[1]) : nullptr;
    a.B = static_cast<int>(B);
    a.S = static_cast<int>(S);
    a.D = D;
    a.half = half_pairing(params) ? 1 : 0;
    a.m = m;
    fill_theta(params, D, a.theta);
    const int rows = 256 / (D / 8);   // four rotation pairs per thread
    for (int side = 0; side < 2; ++side) {
      a.k = static_cast<const uint32_t*>(side == 0 ? k : q);
      a.Hkv = side == 0 ? Hkv : Hq;
      const size_t* off = side == 0 ? lay.off_k : lay.off_q;
      a.k_rot0 = reinterpret_cast<uint32_t*>(ws + off[0]);
      a.k_rot1 = lay.nmaps > 1 ? reinterpret_cast<uint32_t*>(ws + off[1]) : nullptr;
      rope_prep_kernel<<<static_cast<unsigned>((S + rows - 1) / rows), 256, 0, st>>>(a);
      CUDA_TRY(cudaGetLastError(), "backward rope_prep launch");
    }
    for (int i = 0; i < 2; ++i) {
      qm[i] = ws + lay.off_q[lay.nmaps > 1 ? i : 0];
      km[i] = ws + lay.off_k[lay.nmaps > 1 ? i : 0];
    }
    bp.tab0 = a.tab0;
    bp.tab1 = lay.nmaps > 1 ? a.tab1 : a.tab0;
  }
  {
    BwdPrepArgs a{};
    a.dout = static_cast<const __nv_bfloat16*>(dout);
    a.out = out;
    a.lse = lse;
    a.ndelta = reinterpret_cast<float*>(ws + lay.off_delta);
    a.nlse2 = reinterpret_cast<float*>(ws + lay.off_lse2);
    a.B = static_cast<int>(B);
    a.S = static_cast<int>(S);
    a.Hq = Hq;
    a.D = D;
    a.Sp = lay.Sp;
    const long long threads = B * S * Hq * 32;
    bwd_prep_kernel<<<static_cast<unsigned>((threads + 255) / 256), 256, 0, st>>>(a);
    CUDA_TRY(cudaGetLastError(), "backward prep launch");
  }
  // kernel A tiles: 64 query rows, 128 keys; kernel B: 128 query rows, 64 keys
  CUtensorMap ma[6], mb[6];
  if ((rc = make_map(&ma[0], qm[0], D, Hq, S, B, 64, kBwdN, true))) return rc;
  if ((rc = make_map(&ma[1], qm[1], D, Hq, S, B, 64, kBwdN, true))) return rc;
  if ((rc = make_map(&ma[2], km[0], D, Hkv, S, B, 64, kBM, true))) return rc;
  if ((rc = make_map(&ma[3], km[1], D, Hkv, S, B, 64, kBM, true))) return rc;
  if ((rc = make_map(&ma[4], v, D, Hkv, S, B, 64, kBM, true))) return rc;
  if ((rc = make_map(&ma[5], dout, D, Hq, S, B, 64, kBwdN, true))) return rc;
  if ((rc = make_map(&mb[0], qm[0], D, Hq, S, B, 64, kBM, true))) return rc;
  if ((rc = make_map(&mb[1], qm[1], D, Hq, S, B, 64, kBM, true))) return rc;
  if ((rc = make_map(&mb[2], km[0], D, Hkv, S, B, 64, kBwdN, true))) return rc;
  if ((rc = make_map(&mb[3], km[1], D, Hkv, S, B, 64, kBwdN, true))) return rc;
  if ((rc = make_map(&mb[4], v, D, Hkv, S, B, 64, kBwdN, true))) return rc;
  if ((rc = make_map(&mb[5], dout, D, Hq, S, B, 64, kBM, true))) return rc;
  bp.dq = dq;
  bp.dk = dk;
  bp.dv = dv;
  bp.nlse2 = reinterpret_cast<const float*>(ws + lay.off_lse2);
  bp.ndelta = reinterpret_cast<const float*>(ws + lay.off_delta);
  bp.B = static_cast<int>(B);
  bp.S = static_cast<int>(S);
  bp.Hq = Hq;
  bp.Hkv = Hkv;
  bp.Sp = lay.Sp;
  bp.nkt = static_cast<int>(nkt);
  bp.nqt = static_cast<int>(nkt);
  bp.kind = eff;
  bp.window = m.window;
  bp.w0 = m.w0;
  bp.scale_log2 = scale_log2(params, D);
  bp.scale = params->softmax_scale > 0.0f ? params->softmax_scale : static_cast<float>(1.0 / std::sqrt(double(D)));
  bp.half = half_pairing(params) ? 1 : 0;
  const int grid_a = static_cast<int>(nkt * Hkv * B);
  const int grid_b = static_cast<int>(nkt * Hq * B);
  return D == 128 ? launch_backward<128>(ma, mb, bp, grid_a, grid_b, st)
                  : launch_backward<64>(ma, mb, bp, grid_a, grid_b, st);
}
