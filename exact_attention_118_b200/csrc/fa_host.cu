// fa_host.cu - the C ABI declared in include/fa.h: argument checks, TMA
// descriptor encoding, launch configuration and status codes. The whole
// library is this one translation unit (kernels come in through headers).
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "fa.h"
#include "fa_bwd.cuh"
#include "fa_fwd.cuh"

static_assert(fa::kDevErrTimeout == FA_DEVERR_TIMEOUT && fa::kDevErrSmemAlign == FA_DEVERR_SMEM_ALIGN &&
                  fa::kDevErrSeqlens == FA_DEVERR_SEQLENS,
              "device error bits must match the header");

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn g_encode = nullptr;
// Reported by fa_last_cuda_error when a TMA descriptor could not be encoded.
constexpr int kEncodeFailed = -1;
thread_local int t_last_cuda_error = 0;
std::once_flag g_encode_once;

EncodeTiledFn encode_fn() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  });
  return g_encode;
}

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);
CtxGetCurrentFn g_ctx_current = nullptr;
CtxGetIdFn g_ctx_id = nullptr;
std::once_flag g_ctx_once;

// The unique ID of the CUDA context current on this thread, 0 if there is
// none. The driver never reuses a context ID within a process, so state kept
// under one ID is never taken for state of a later context (one created after
// cudaDeviceReset, or one the caller made current through the driver API).
unsigned long long current_ctx_id() {
  std::call_once(g_ctx_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_current = reinterpret_cast<CtxGetCurrentFn>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_id = reinterpret_cast<CtxGetIdFn>(fn);
  });
  if (!g_ctx_current || !g_ctx_id) return 0;
  CUcontext c = nullptr;
  if (g_ctx_current(&c) != CUDA_SUCCESS || c == nullptr) return 0;
  unsigned long long id = 0;
  return g_ctx_id(c, &id) == CUDA_SUCCESS ? id : 0;
}

// A small table of values kept per CUDA context: the results of one-time
// set-up steps. Up to kSlots contexts; past that the oldest entry is reused.
template <typename T>
class PerContext {
 public:
  bool get(unsigned long long id, T* out) {
    if (id == 0) return false;
    std::lock_guard<std::mutex> lock(mu_);
    for (int i = 0; i < n_; ++i)
      if (ids_[i] == id) {
        *out = vals_[i];
        return true;
      }
    return false;
  }
  void put(unsigned long long id, T v) {
    if (id == 0) return;
    std::lock_guard<std::mutex> lock(mu_);
    for (int i = 0; i < n_; ++i)
      if (ids_[i] == id) {
        vals_[i] = v;
        return;
      }
    const int slot = n_ < kSlots ? n_++ : (next_++ % kSlots);
    ids_[slot] = id;
    vals_[slot] = v;
  }

 private:
  static constexpr int kSlots = 16;
  std::mutex mu_;
  unsigned long long ids_[kSlots] = {};
  T vals_[kSlots] = {};
  int n_ = 0, next_ = 0;
};

// A kernel's dynamic shared memory limit is raised once per context, not on
// every launch. The caller keeps one table per kernel instantiation.
template <typename Kern>
fa_status set_smem_once(PerContext<int>& done, Kern kern, int smem) {
  int have = 0;
  if (done.get(current_ctx_id(), &have) && have == smem) return FA_OK;
  if (cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) {
    t_last_cuda_error = static_cast<int>(e);
    return FA_ERR_CUDA;
  }
  done.put(current_ctx_id(), smem);  // the call above makes a context current if none was
  return FA_OK;
}

constexpr int kMaxDevices = 64;

// Streaming multiprocessors of the current device, cached per device.
int sm_count() {
  static std::atomic<int> cache[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  const bool slot = dev >= 0 && dev < kMaxDevices;
  if (slot) {
    const int v = cache[dev].load(std::memory_order_relaxed);
    if (v > 0) return v;
  }
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) sms = 148;
  if (slot) cache[dev].store(sms, std::memory_order_relaxed);
  return sms;
}

// The kernels use tcgen05 and TMA: compute capability 10.0 (sm_100a) only.
fa_status check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return FA_ERR_CUDA;
  if (major != 10 || minor != 0) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

fa_status check_sizes(int B, int H, int N, int d, float scale, int causal) {
  if (B < 1 || H < 1 || N < 1 || d < 1) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (!(std::isfinite(scale) && scale > 0.f)) return FA_ERR_INVALID_ARG;
  const long long rows = static_cast<long long>(B) * H * N;
  if (rows >= (1ll << 31)) return FA_ERR_INVALID_ARG;
  // Tile and band bounds are formed in 32-bit ints (up to about 2 N).
  if (N > (1 << 29)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

// Where the rows of one call live. Fixed length: [B, heads, N, inner]
// tensors, seen by TMA as dims {inner, N, B*heads}. Packed variable length:
// [T, heads, inner] tensors holding sequence b in rows [cu[b], cu[b+1]), seen
// as dims {inner, T, heads} (the head stride is then the smaller one). Either
// way a tile is (column, row, head) and out-of-range rows read as zero and are
// clipped on store, so a ragged tile never touches the next head.
struct Geom {
  int B, H, Hkv, N;         // N: the sequence length (the longest, if packed)
  int T = 0;                // packed rows
  const int* cu = nullptr;  // packed: [B + 1] prefix sums of the lengths (device)
  bool packed() const { return cu != nullptr; }
  int rows() const { return packed() ? T : N; }  // row dimension of every map
  int map_heads(int heads) const { return packed() ? heads : B * heads; }
};

// Encoded tensor maps, cached. A map is a pure function of its encoding
// arguments (address, sizes, strides, box, type, swizzle), so a cached map
// equals a fresh encoding of the same arguments whatever happened to the
// memory in between; the cache only saves the host time of encoding (the
// calls encode 4 to 9 maps each). Direct-mapped by a hash of the key.
struct MapKey {
  const void* base;
  cuuint64_t dims[3], strides[2];
  cuuint32_t box[3];
  int rank, dtype, swizzle;
  bool operator==(const MapKey& o) const { return std::memcmp(this, &o, sizeof(MapKey)) == 0; }
};

class MapCache {
 public:
  // Encodes (or finds) the map; the result is copied out under the lock.
  CUresult get(const MapKey& key, CUtensorMap* out) {
    uint64_t h = 1469598103934665603ull;  // FNV-1a over the key bytes
    const unsigned char* b = reinterpret_cast<const unsigned char*>(&key);
    for (size_t i = 0; i < sizeof(MapKey); ++i) h = (h ^ b[i]) * 1099511628211ull;
    const size_t slot = static_cast<size_t>(h % kSlots);
    std::lock_guard<std::mutex> lock(mu_);
    if (valid_[slot] && keys_[slot] == key) {
      *out = maps_[slot];
      return CUDA_SUCCESS;
    }
    EncodeTiledFn enc = encode_fn();
    if (!enc) return CUDA_ERROR_NOT_INITIALIZED;
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    CUresult r = enc(&maps_[slot], static_cast<CUtensorMapDataType>(key.dtype), static_cast<cuuint32_t>(key.rank),
                     const_cast<void*>(key.base), key.dims, key.strides, key.box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, static_cast<CUtensorMapSwizzle>(key.swizzle),
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    valid_[slot] = (r == CUDA_SUCCESS);
    if (r != CUDA_SUCCESS) return r;
    keys_[slot] = key;
    *out = maps_[slot];
    return CUDA_SUCCESS;
  }

 private:
  static constexpr size_t kSlots = 256;
  std::mutex mu_;
  MapKey keys_[kSlots];
  alignas(64) CUtensorMap maps_[kSlots];
  bool valid_[kSlots] = {};
};
MapCache g_maps;

fa_status encode_map(CUtensorMap* m, const MapKey& key) {
  if (!encode_fn()) return FA_ERR_CUDA;
  const CUresult r = g_maps.get(key, m);
  if (r != CUDA_SUCCESS) t_last_cuda_error = kEncodeFailed;
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

fa_status make_head_map(CUtensorMap* m, const void* base, const Geom& g, int heads, CUtensorMapDataType dt,
                        int elem_bytes, int inner, int box_inner, int box_rows, CUtensorMapSwizzle sw) {
  const cuuint64_t row_bytes = static_cast<cuuint64_t>(inner) * elem_bytes;
  MapKey key{};
  key.base = base;
  key.dims[0] = static_cast<cuuint64_t>(inner);
  key.dims[1] = static_cast<cuuint64_t>(g.rows());
  key.dims[2] = static_cast<cuuint64_t>(g.map_heads(heads));
  key.strides[0] = g.packed() ? row_bytes * heads : row_bytes;
  key.strides[1] = g.packed() ? row_bytes : row_bytes * g.N;
  key.box[0] = static_cast<cuuint32_t>(box_inner);
  key.box[1] = static_cast<cuuint32_t>(box_rows);
  key.box[2] = 1u;
  key.rank = 3;
  key.dtype = static_cast<int>(dt);
  key.swizzle = static_cast<int>(sw);
  return encode_map(m, key);
}

// bf16 tiles of 128 rows x 64 columns (128-byte swizzle).
fa_status make_bf16_tile_map(CUtensorMap* m, const void* base, const Geom& g, int heads, int d) {
  return make_head_map(m, base, g, heads, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, 64, 128,
                       CU_TENSOR_MAP_SWIZZLE_128B);
}

// bf16 output rows in 32-row boxes of 64 columns (128-byte swizzle): the
// per-warp TMA stores of O, dK and dV.
fa_status make_out_map(CUtensorMap* m, const void* base, const Geom& g, int heads, int d) {
  return make_head_map(m, base, g, heads, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, 64, 32,
                       CU_TENSOR_MAP_SWIZZLE_128B);
}

// Caller-provided events recorded around the main backward kernel
// (fa_set_bwd_main_events); per host thread.
thread_local cudaEvent_t t_bwd_ev_before = nullptr;
thread_local cudaEvent_t t_bwd_ev_after = nullptr;

fa_status launch_status() {
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) return FA_OK;
  t_last_cuda_error = static_cast<int>(e);
  return FA_ERR_CUDA;
}

fa_status cuda_fail(cudaError_t e) {
  t_last_cuda_error = static_cast<int>(e);
  return FA_ERR_CUDA;
}

// Grid for the memory-bound helper kernels: enough CTAs to fill every SM a
// few times over, grid-striding beyond that.
unsigned helper_grid(long long threads_needed) {
  const int sms = sm_count();
  const long long blocks = (threads_needed + 255) / 256;
  const long long cap = static_cast<long long>(sms) * 8;
  return static_cast<unsigned>(blocks < 1 ? 1 : (blocks < cap ? blocks : cap));
}

// Causal grids launch the heaviest tiles first, which spreads the CTAs that
// run at the same time over many heads. Splitting the heads (units) into
// groups, heaviest-first within each, keeps a group's streamed operands in L2
// (about 64 MB of its 126 MB). A group must also hold enough work that its
// heaviest CTA (about 2 tiles' worth of steps per tile of the longest axis)
// finishes no later than the group's other CTAs: with `tiles` tiles per unit
// and work ~ tiles^2 per unit spread over the SMs, that needs a group of at
// least 2 * SMs / tiles units. A working set within one group's budget keeps
// one group: the global heaviest-first order. Returns the number of groups.
int sched_groups(long long bytes_per_unit, int units, int tiles) {
  const long long budget = 64ll << 20;  // streamed operands of one group
  if (bytes_per_unit * units <= budget) return 1;
  const int sms = sm_count();
  long long g_max = bytes_per_unit > 0 ? budget / bytes_per_unit : units;
  if (g_max < 1) g_max = 1;
  long long g_min = tiles > 0 ? (2ll * sms + tiles - 1) / tiles : 1;
  if (g_min < 1) g_min = 1;
  long long groups = (units + g_max - 1) / g_max;  // fit in L2
  const long long most = units / g_min;            // no group below g_min
  if (groups > most) groups = most;
  if (groups < 1) groups = 1;
  if (groups > units) groups = units;
  return static_cast<int>(groups);
}

// The mask a call asks for, reduced to one of the kernels' three modes. A
// window wider than the sequence on a side is no bound on that side, so a
// band that bounds nothing is the unmasked kernel and a band bounded only on
// the right at 0 is the causal one.
struct Mask {
  int mode, wl, wr;
};
Mask resolve_mask(int wl, int wr, int N) {
  const int l = (wl < 0 || wl >= N - 1) ? N : wl;
  const int r = (wr < 0 || wr >= N - 1) ? N : wr;
  if (l == N && r == N) return {fa::kMaskNone, 0, 0};
  if (l == N && r == 0) return {fa::kMaskCausal, 0, 0};
  return {fa::kMaskBand, l, r};
}

template <int D, int MASK, bool OF32, bool FP8 = false>
fa_status launch_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& to,
                     const fa::FwdParams& p, cudaStream_t st) {
  auto kern = fa::fa_fwd_kernel<D, MASK, OF32, FP8>;
  const int smem = fa::FwdLayout<D, FP8 ? 1 : 2>::kAlloc;
  static PerContext<int> attr_set;
  if (fa_status s = set_smem_once(attr_set, kern, smem)) return s;
  const unsigned grid = static_cast<unsigned>(p.n_pairs) * static_cast<unsigned>(p.BH);
  kern<<<grid, fa::kFwdThreads, smem, st>>>(tq, tk, tv, to, p);
  return launch_status();
}

template <int D, bool OF32, bool FP8 = false>
fa_status launch_fwd_mask(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& to,
                          const fa::FwdParams& p, int mode, cudaStream_t st) {
  if (mode == fa::kMaskCausal) return launch_fwd<D, fa::kMaskCausal, OF32, FP8>(tq, tk, tv, to, p, st);
  if (mode == fa::kMaskBand) return launch_fwd<D, fa::kMaskBand, OF32, FP8>(tq, tk, tv, to, p, st);
  return launch_fwd<D, fa::kMaskNone, OF32, FP8>(tq, tk, tv, to, p, st);
}

// 2-D fp32 map of a [BH][Np] statistics array (Np >= N, a multiple of 4),
// dims {N, BH}: a 128-wide row box (one query tile), zero-filled past N.
fa_status make_stat_map(CUtensorMap* m, const float* base, int N, int Np, int BH) {
  MapKey key{};
  key.base = base;
  key.dims[0] = static_cast<cuuint64_t>(N);
  key.dims[1] = static_cast<cuuint64_t>(BH);
  key.strides[0] = static_cast<cuuint64_t>(Np) * 4;
  key.box[0] = 128u;
  key.box[1] = 1u;
  key.rank = 2;
  key.dtype = static_cast<int>(CU_TENSOR_MAP_DATA_TYPE_FLOAT32);
  key.swizzle = static_cast<int>(CU_TENSOR_MAP_SWIZZLE_NONE);
  return encode_map(m, key);
}

template <int D, int MASK>
fa_status launch_bwd_main(const CUtensorMap* maps, const fa::BwdParams& p, cudaStream_t st) {
  auto kern = fa::fa_bwd_kernel<D, MASK>;
  const int smem = fa::BwdLayout<D>::kAlloc;
  static PerContext<int> attr_set;
  if (fa_status s = set_smem_once(attr_set, kern, smem)) return s;
  const unsigned grid = static_cast<unsigned>(p.n_kv) * static_cast<unsigned>(p.BH);
  if (t_bwd_ev_before && cudaEventRecord(t_bwd_ev_before, st) != cudaSuccess) return FA_ERR_CUDA;
  kern<<<grid, fa::kBwdThreads, smem, st>>>(maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], maps[6], maps[7],
                                            maps[8], p);
  const fa_status s = launch_status();
  if (s == FA_OK && t_bwd_ev_after && cudaEventRecord(t_bwd_ev_after, st) != cudaSuccess) return FA_ERR_CUDA;
  return s;
}

// How many CTAs share one K/V head's query heads in the backward (a divisor
// of the group size H / Hkv; 1 for multi-head attention). One CTA per
// (K/V head, key tile) keeps dK and dV on chip for the whole group, but a few
// K/V heads give too few CTAs to fill the GPU, and causal key tiles differ
// in cost. So take the smallest divisor that gives at least 8 CTAs per SM
// (the whole group when none does); shares then add their partial dK and dV
// in fp32 global memory.
int bwd_split(int B, int H, int Hkv, int N) {
  const int group = H / Hkv;
  if (group == 1) return 1;
  const int sms = sm_count();
  const long long base = static_cast<long long>((N + 127) / 128) * B * Hkv;
  for (int s = 1; s < group; ++s)
    if (group % s == 0 && base * s >= 8LL * sms) return s;
  return group;
}

template <int D>
fa_status launch_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                     void* dq, void* dk, void* dv, void* workspace, const Geom& g, float scale, Mask mask,
                     cudaStream_t st) {
  // Workspace rows: the row dimension Nr of the maps times their head count.
  const int Nr = g.rows(), BHr = g.map_heads(g.H), BHkvr = g.map_heads(g.Hkv);
  const long long rows = static_cast<long long>(BHr) * Nr;
  // Statistics row length: N rounded up to 4, or the packed per-sequence
  // layout of fa::varlen_stat_stride.
  const int Np = g.packed() ? fa::varlen_stat_stride(g.T, g.B) : fa::stat_stride(Nr);
  const size_t stat_bytes = fa::align256(static_cast<size_t>(BHr) * Np * sizeof(float));
  char* ws = static_cast<char*>(workspace);
  float* dq_acc = reinterpret_cast<float*>(ws);
  float* lse2 = reinterpret_cast<float*>(ws + fa::align256(rows * D * sizeof(float)));
  float* dsum = reinterpret_cast<float*>(reinterpret_cast<char*>(lse2) + stat_bytes);
  const int n_split = bwd_split(g.B, g.H, g.Hkv, g.N);
  float* dk_acc = nullptr;
  float* dv_acc = nullptr;
  const long long kv_elems = static_cast<long long>(BHkvr) * Nr * D;
  const size_t kv_acc_bytes = fa::bwd_kv_acc_bytes(1, BHkvr, Nr, D);
  if (n_split > 1) {
    dk_acc = reinterpret_cast<float*>(reinterpret_cast<char*>(dsum) + stat_bytes);
    dv_acc = reinterpret_cast<float*>(reinterpret_cast<char*>(dk_acc) + kv_acc_bytes);
  }

  // 1. D = rowsum(dO * O), lse2 = lse * log2(e), dQ (and split dK/dV) accumulators = 0.
  const long long kv_n4 = n_split > 1 ? static_cast<long long>(2 * kv_acc_bytes) / 16 : 0;
  if (g.packed()) {
    // One grid row per sequence (strided past 65535), enough blocks across
    // for the longest sequence, the total kept to a few waves.
    const int gy = g.B < 65535 ? g.B : 65535;
    long long gx = (static_cast<long long>(g.N) * g.H * (D / 8) + 255) / 256;
    const long long cap = (static_cast<long long>(helper_grid(1LL << 40)) * 2 + gy - 1) / gy;
    gx = gx < cap ? gx : cap;
    fa::fa_bwd_dot_varlen_kernel<D><<<dim3(static_cast<unsigned>(gx < 1 ? 1 : gx), gy), 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dO), lse, lse2, dsum, dq_acc, g.cu,
        g.B, g.T, g.H, g.N, Np, dk_acc, kv_n4);
  } else {
    fa::fa_bwd_dot_kernel<D><<<helper_grid(rows * (D / 8)), 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dO), lse, lse2, dsum, dq_acc, rows,
        Nr, Np, dk_acc, kv_n4);
  }
  fa_status s = launch_status();
  if (s != FA_OK) return s;

  // 2. Main kernel. Maps: q, k, v, dO (128-row tiles), dQ accumulator (fp32,
  // 32-row box), lse2, D, and the dK, dV outputs (32-row boxes; bf16, or the
  // fp32 accumulators when query heads are split across CTAs).
  alignas(64) CUtensorMap maps[9];
  if ((s = make_bf16_tile_map(&maps[0], q, g, g.H, D)) != FA_OK) return s;
  if ((s = make_bf16_tile_map(&maps[1], k, g, g.Hkv, D)) != FA_OK) return s;
  if ((s = make_bf16_tile_map(&maps[2], v, g, g.Hkv, D)) != FA_OK) return s;
  if ((s = make_bf16_tile_map(&maps[3], dO, g, g.H, D)) != FA_OK) return s;
  if ((s = make_head_map(&maps[4], dq_acc, g, g.H, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, D, D, 32,
                         CU_TENSOR_MAP_SWIZZLE_NONE)) != FA_OK)
    return s;
  const int stat_dim = g.packed() ? Np : Nr;
  if ((s = make_stat_map(&maps[5], lse2, stat_dim, Np, BHr)) != FA_OK) return s;
  if ((s = make_stat_map(&maps[6], dsum, stat_dim, Np, BHr)) != FA_OK) return s;
  for (int t = 0; t < 2; ++t) {
    const void* out = n_split > 1 ? static_cast<const void*>(t ? dv_acc : dk_acc) : (t ? dv : dk);
    s = n_split > 1 ? make_head_map(&maps[7 + t], out, g, g.Hkv, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, D, 32, 32,
                                    CU_TENSOR_MAP_SWIZZLE_128B)
                    : make_out_map(&maps[7 + t], out, g, g.Hkv, D);
    if (s != FA_OK) return s;
  }
  fa::BwdParams p;
  p.dk = dk;
  p.dv = dv;
  p.dk_acc = dk_acc;
  p.dv_acc = dv_acc;
  p.BH = g.B * g.Hkv * n_split;
  p.H = g.H;
  p.Hkv = g.Hkv;
  p.n_split = n_split;
  p.wl = mask.wl;
  p.wr = mask.wr;
  // Per unit: Q and dO (bf16) and the fp32 dQ accumulator of its query heads.
  p.sched_groups = sched_groups(static_cast<long long>(g.H / g.Hkv / n_split) * g.N * D * 8, p.BH, (g.N + 127) / 128);
  p.cu_seqlens = g.cu;
  p.T = g.T;
  p.N = g.N;
  p.n_kv = (g.N + 127) / 128;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  s = mask.mode == fa::kMaskCausal ? launch_bwd_main<D, fa::kMaskCausal>(maps, p, st)
      : mask.mode == fa::kMaskBand ? launch_bwd_main<D, fa::kMaskBand>(maps, p, st)
                                   : launch_bwd_main<D, fa::kMaskNone>(maps, p, st);
  if (s != FA_OK) return s;

  // 3. dq = bf16(dQ accumulator).
  const long long n8 = rows * D / 8;
  fa::fa_bwd_dq_convert_kernel<<<helper_grid(n8), 256, 0, st>>>(dq_acc, static_cast<__nv_bfloat16*>(dq), n8);
  if ((s = launch_status()) != FA_OK || n_split == 1) return s;

  // 4. Split grouped-query heads: dk, dv = bf16(their fp32 accumulators).
  fa::fa_bwd_dq_convert_kernel<<<helper_grid(kv_elems / 8), 256, 0, st>>>(
      dk_acc, static_cast<__nv_bfloat16*>(dk), kv_elems / 8);
  if ((s = launch_status()) != FA_OK) return s;
  fa::fa_bwd_dq_convert_kernel<<<helper_grid(kv_elems / 8), 256, 0, st>>>(
      dv_acc, static_cast<__nv_bfloat16*>(dv), kv_elems / 8);
  return launch_status();
}

// Failure-detection self-test: one thread waits, through the same bounded
// wait the kernels use, on an mbarrier that nothing ever completes. The wait
// gives up after its time limit, records a timeout in the device error
// word and the kernel returns normally.
__global__ void fa_selftest_wait_kernel() {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    fa::mbar_init(&bar, 1);
    abort_flag = 0;
    fa::fence_barrier_init();
    fa::wait_parity(&bar, 0, &abort_flag);
  }
}

// ---------------------------------------------------------------------------
// Fixed scratch for fa_bwd_noalloc. Some callers may not allocate device
// memory at all: code that runs inside a host application which owns every
// GPU allocation (a plug-in handed only its tensors), or a latency-critical
// path where a cudaMalloc's unpredictable cost is not allowed. For them the
// backward's workspace lives in this file-scope device array instead. Every
// GPU that loads the library holds it (FA_NOALLOC_SCRATCH_BYTES) until exit.
// In host code the array's name is only a stand-in, not a device address:
// its address comes from cudaGetSymbolAddress, taken with the device current
// and cached per CUDA context. The address belongs to the context, so a new
// context on the same device (after cudaDeviceReset, or a driver-API context
// the caller made current) takes its own.
static __device__ __align__(256) unsigned char g_noalloc_scratch[FA_NOALLOC_SCRATCH_BYTES];

PerContext<void*> g_noalloc_addr;

fa_status noalloc_scratch(void** out) {
  void* addr = nullptr;
  if (g_noalloc_addr.get(current_ctx_id(), &addr) && addr != nullptr) {
    *out = addr;
    return FA_OK;
  }
  if (cudaError_t e = cudaGetSymbolAddress(&addr, g_noalloc_scratch)) return cuda_fail(e);
  g_noalloc_addr.put(current_ctx_id(), addr);  // the lookup makes a context current if none was
  *out = addr;
  return FA_OK;
}

// The forward for either layout; arguments already checked.
fa_status fwd_impl(const Geom& g, const void* q, const void* k, const void* v, void* o, float* lse, int d,
                   float scale, int window_left, int window_right, fa_dtype o_dtype, void* stream) {
  fa_status s;
  alignas(64) CUtensorMap tq, tk, tv, to;
  if ((s = make_bf16_tile_map(&tq, q, g, g.H, d)) != FA_OK) return s;
  if ((s = make_bf16_tile_map(&tk, k, g, g.Hkv, d)) != FA_OK) return s;
  if ((s = make_bf16_tile_map(&tv, v, g, g.Hkv, d)) != FA_OK) return s;
  // bf16 O, stored by TMA in 32-row boxes (an fp32 O is written by the
  // threads; the map is then unused).
  if ((s = make_out_map(&to, o, g, g.H, d)) != FA_OK) return s;

  fa::FwdParams p;
  p.o = o;
  p.lse = lse;
  p.BH = g.B * g.H;
  p.H = g.H;
  p.Hkv = g.Hkv;
  p.N = g.N;
  p.n_pairs = (g.N + 255) / 256;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.o_scale = 1.f;
  p.sched_groups = sched_groups(2ll * g.N * d * 2, g.B * g.H, p.n_pairs);  // K and V of a head, bf16
  const Mask m = resolve_mask(window_left, window_right, g.N);
  p.wl = m.wl;
  p.wr = m.wr;
  p.cu_seqlens = g.cu;
  p.T = g.T;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool f32 = (o_dtype == FA_F32);
  if (d == 64)
    return f32 ? launch_fwd_mask<64, true>(tq, tk, tv, to, p, m.mode, st)
               : launch_fwd_mask<64, false>(tq, tk, tv, to, p, m.mode, st);
  return f32 ? launch_fwd_mask<128, true>(tq, tk, tv, to, p, m.mode, st)
             : launch_fwd_mask<128, false>(tq, tk, tv, to, p, m.mode, st);
}

// The FP8 forward (fixed-length layout, D = 128); arguments already checked.
fa_status fwd_fp8_impl(const Geom& g, const void* q8, const void* k8, const void* v8, void* o, float* lse,
                       float scale, float q_scale, float k_scale, float v_scale, int window_left, int window_right,
                       fa_dtype o_dtype, void* stream) {
  fa_status s;
  alignas(64) CUtensorMap tq, tk, tv, to;
  const auto u8 = CU_TENSOR_MAP_DATA_TYPE_UINT8;
  if ((s = make_out_map(&to, o, g, g.H, 128)) != FA_OK) return s;  // unused: the FP8 kernel's threads write O
  if ((s = make_head_map(&tq, q8, g, g.H, u8, 1, 128, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK) return s;
  if ((s = make_head_map(&tk, k8, g, g.Hkv, u8, 1, 128, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK) return s;
  if ((s = make_head_map(&tv, v8, g, g.Hkv, u8, 1, 128, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK) return s;
  fa::FwdParams p;
  p.o = o;
  p.lse = lse;
  p.BH = g.B * g.H;
  p.H = g.H;
  p.Hkv = g.Hkv;
  p.N = g.N;
  p.n_pairs = (g.N + 255) / 256;
  p.scale_log2 = scale * q_scale * k_scale * 1.4426950408889634f;
  p.o_scale = v_scale;
  p.sched_groups = sched_groups(2ll * g.N * 128, g.B * g.H, p.n_pairs);  // K and V of a head, e4m3
  const Mask m = resolve_mask(window_left, window_right, g.N);
  p.wl = m.wl;
  p.wr = m.wr;
  p.cu_seqlens = g.cu;
  p.T = g.T;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return o_dtype == FA_F32 ? launch_fwd_mask<128, true, true>(tq, tk, tv, to, p, m.mode, st)
                           : launch_fwd_mask<128, false, true>(tq, tk, tv, to, p, m.mode, st);
}

// The backward for either layout; arguments already checked.
fa_status bwd_impl(const Geom& g, const void* q, const void* k, const void* v, const void* o, const float* lse,
                   const void* dO, void* dq, void* dk, void* dv, void* workspace, int d, float scale,
                   int window_left, int window_right, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Mask m = resolve_mask(window_left, window_right, g.N);
  if (d == 64) return launch_bwd<64>(q, k, v, o, lse, dO, dq, dk, dv, workspace, g, scale, m, st);
  return launch_bwd<128>(q, k, v, o, lse, dO, dq, dk, dv, workspace, g, scale, m, st);
}

// Checks shared by the variable-length calls: the prefix-sum array, the head
// grouping and the sizes (T packed rows of H heads within int range).
fa_status check_varlen(const int* cu_seqlens, int B, int max_seqlen, int T, int H, int Hkv, int d, float scale) {
  if (cu_seqlens == nullptr || (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0) return FA_ERR_INVALID_ARG;
  if (max_seqlen < 1) return FA_ERR_INVALID_ARG;
  fa_status s = check_sizes(1, H, T, d, scale, 0);
  if (s != FA_OK) return s;
  if (B < 1 || Hkv < 1 || H % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H >= (1ll << 31)) return FA_ERR_INVALID_ARG;
  if ((static_cast<long long>(T) + 4LL * B + 8) * H >= (1ll << 31)) return FA_ERR_INVALID_ARG;
  return FA_OK;
}

// Test hook: y = exp2_fma2(x), the forward's FMA-pipe exp2, element by
// element (pairs; an odd last element is paired with itself).
__global__ void fa_selftest_exp2_kernel(const float* __restrict__ x, float* __restrict__ y, long long n) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = 2 * (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x); i < n; i += 2 * stride) {
    const bool pair = i + 1 < n;
    const float2 r = fa::exp2_fma2(make_float2(x[i], pair ? x[i + 1] : x[i]));
    y[i] = r.x;
    if (pair) y[i + 1] = r.y;
  }
}

}  // namespace

extern "C" {

int fa_version(void) { return 100; }

const char* fa_strerror(fa_status s) {
  switch (s) {
    case FA_OK: return "success";
    case FA_ERR_INVALID_ARG: return "invalid argument";
    case FA_ERR_UNSUPPORTED: return "unsupported configuration or device";
    case FA_ERR_CUDA: return "CUDA error";
    case FA_ERR_TIMEOUT: return "a bounded device-side wait timed out";
  }
  return "unknown status";
}

fa_status fa_fwd_window(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Hkv,
                        int N, int d, float scale, int window_left, int window_right, fa_dtype o_dtype,
                        void* stream) {
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return FA_ERR_INVALID_ARG;
  if (o_dtype != FA_BF16 && o_dtype != FA_F32) return FA_ERR_INVALID_ARG;
  fa_status s = check_sizes(B, H, N, d, scale, 0);
  if (s != FA_OK) return s;
  if (Hkv < 1 || H % Hkv != 0) return FA_ERR_INVALID_ARG;
  if ((s = check_device()) != FA_OK) return s;
  return fwd_impl(Geom{B, H, Hkv, N}, q, k, v, o, lse, d, scale, window_left, window_right, o_dtype, stream);
}

fa_status fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse, const int* cu_seqlens,
                        int B, int max_seqlen, int T, int H, int Hkv, int d, float scale, int window_left,
                        int window_right, fa_dtype o_dtype, void* stream) {
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return FA_ERR_INVALID_ARG;
  if (o_dtype != FA_BF16 && o_dtype != FA_F32) return FA_ERR_INVALID_ARG;
  fa_status s = check_varlen(cu_seqlens, B, max_seqlen, T, H, Hkv, d, scale);
  if (s != FA_OK) return s;
  if ((s = check_device()) != FA_OK) return s;
  Geom g{B, H, Hkv, max_seqlen < T ? max_seqlen : T};
  g.T = T;
  g.cu = cu_seqlens;
  return fwd_impl(g, q, k, v, o, lse, d, scale, window_left, window_right, o_dtype, stream);
}

fa_status fa_fwd_fp8(const void* q8, const void* k8, const void* v8, void* o, float* lse, int B, int H, int Hkv,
                     int N, int d, float scale, float q_scale, float k_scale, float v_scale, int window_left,
                     int window_right, fa_dtype o_dtype, void* stream) {
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(v8) || !aligned16(o) || !aligned16(lse))
    return FA_ERR_INVALID_ARG;
  if (o_dtype != FA_BF16 && o_dtype != FA_F32) return FA_ERR_INVALID_ARG;
  fa_status s = check_sizes(B, H, N, d, scale, 0);
  if (s != FA_OK) return s;
  if (Hkv < 1 || H % Hkv != 0) return FA_ERR_INVALID_ARG;
  for (float x : {q_scale, k_scale, v_scale})
    if (!(std::isfinite(x) && x > 0.f)) return FA_ERR_INVALID_ARG;
  if (d != 128) return FA_ERR_UNSUPPORTED;
  if ((s = check_device()) != FA_OK) return s;
  return fwd_fp8_impl(Geom{B, H, Hkv, N}, q8, k8, v8, o, lse, scale, q_scale, k_scale, v_scale, window_left,
                      window_right, o_dtype, stream);
}

fa_status fa_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Hkv,
                     int N, int d, float scale, int causal, fa_dtype o_dtype, void* stream) {
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  return fa_fwd_window(q, k, v, o, lse, B, H, Hkv, N, d, scale, -1, causal ? 0 : -1, o_dtype, stream);
}

size_t fa_bwd_workspace_size(int B, int H, int N, int d) {
  if (check_sizes(B, H, N, d, 1.f, 0) != FA_OK) return 0;
  return fa::bwd_workspace_bytes(B * H, N, d);
}

size_t fa_bwd_gqa_workspace_size(int B, int H, int Hkv, int N, int d) {
  if (check_sizes(B, H, N, d, 1.f, 0) != FA_OK || Hkv < 1 || H % Hkv != 0) return 0;
  return fa::bwd_gqa_workspace_bytes(B, H, Hkv, N, d);
}

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
                 float scale, int causal, fa_dtype o_dtype, void* stream) {
  return fa_fwd_gqa(q, k, v, o, lse, B, H, H, N, d, scale, causal, o_dtype, stream);
}

fa_status fa_bwd_window(const void* q, const void* k, const void* v, const void* o, const float* lse,
                        const void* dO, void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes, int B, int H,
                        int Hkv, int N, int d, float scale, int window_left, int window_right, void* stream) {
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) || !aligned16(dO) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return FA_ERR_INVALID_ARG;
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return FA_ERR_INVALID_ARG;
  fa_status s = check_sizes(B, H, N, d, scale, 0);
  if (s != FA_OK) return s;
  if (Hkv < 1 || H % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (ws_bytes < fa::bwd_gqa_workspace_bytes(B, H, Hkv, N, d)) return FA_ERR_INVALID_ARG;
  if ((s = check_device()) != FA_OK) return s;
  return bwd_impl(Geom{B, H, Hkv, N}, q, k, v, o, lse, dO, dq, dk, dv, workspace, d, scale, window_left,
                  window_right, stream);
}

size_t fa_bwd_varlen_workspace_size(int B, int T, int H, int Hkv, int d) {
  if (B < 1 || check_sizes(1, H, T, d, 1.f, 0) != FA_OK || Hkv < 1 || H % Hkv != 0) return 0;
  if ((static_cast<long long>(T) + 4LL * B + 8) * H >= (1ll << 31)) return 0;
  return fa::bwd_varlen_workspace_bytes(B, T, H, Hkv, d);
}

fa_status fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const float* lse,
                        const void* dO, void* dq, void* dk, void* dv, const int* cu_seqlens, void* workspace,
                        size_t ws_bytes, int B, int max_seqlen, int T, int H, int Hkv, int d, float scale,
                        int window_left, int window_right, void* stream) {
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) || !aligned16(dO) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return FA_ERR_INVALID_ARG;
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return FA_ERR_INVALID_ARG;
  fa_status s = check_varlen(cu_seqlens, B, max_seqlen, T, H, Hkv, d, scale);
  if (s != FA_OK) return s;
  if (ws_bytes < fa::bwd_varlen_workspace_bytes(B, T, H, Hkv, d)) return FA_ERR_INVALID_ARG;
  if ((s = check_device()) != FA_OK) return s;
  Geom g{B, H, Hkv, max_seqlen < T ? max_seqlen : T};
  g.T = T;
  g.cu = cu_seqlens;
  return bwd_impl(g, q, k, v, o, lse, dO, dq, dk, dv, workspace, d, scale, window_left, window_right, stream);
}

fa_status fa_bwd_gqa(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                     void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes, int B, int H, int Hkv, int N,
                     int d, float scale, int causal, void* stream) {
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  return fa_bwd_window(q, k, v, o, lse, dO, dq, dk, dv, workspace, ws_bytes, B, H, Hkv, N, d, scale, -1,
                       causal ? 0 : -1, stream);
}

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                 void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes, int B, int H, int N, int d,
                 float scale, int causal, void* stream) {
  return fa_bwd_gqa(q, k, v, o, lse, dO, dq, dk, dv, workspace, ws_bytes, B, H, H, N, d, scale, causal, stream);
}

int fa_last_cuda_error(void) { return t_last_cuda_error; }

fa_status fa_selftest_wait_timeout(void* stream) {
  fa_status s = check_device();
  if (s != FA_OK) return s;
  fa_selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>();
  return launch_status();
}

fa_status fa_selftest_exp2_fma(const float* x, float* y, long long n, void* stream) {
  if (n < 0 || (n > 0 && (x == nullptr || y == nullptr))) return FA_ERR_INVALID_ARG;
  if (n == 0) return FA_OK;
  fa_status s = check_device();
  if (s != FA_OK) return s;
  fa_selftest_exp2_kernel<<<helper_grid((n + 1) / 2), 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n);
  return launch_status();
}

fa_status fa_set_bwd_main_events(void* before, void* after) {
  t_bwd_ev_before = static_cast<cudaEvent_t>(before);
  t_bwd_ev_after = static_cast<cudaEvent_t>(after);
  return FA_OK;
}

fa_status fa_decode_device_error(unsigned int word) {
  if (word == 0u) return FA_OK;
  if (word & FA_DEVERR_TIMEOUT) return FA_ERR_TIMEOUT;
  if (word & ~FA_DEVERR_SEQLENS) return FA_ERR_CUDA;  // FA_DEVERR_SMEM_ALIGN or an unknown bit
  return FA_ERR_INVALID_ARG;                               // malformed cu_seqlens, clamped by the kernels
}

fa_status fa_get_device_error(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaError_t e = cudaStreamSynchronize(st)) return cuda_fail(e);
  unsigned int word = 0u;
  if (cudaError_t e = cudaMemcpyFromSymbol(&word, fa::g_device_error, sizeof(word))) return cuda_fail(e);
  if (word != 0u) {
    const unsigned int zero = 0u;
    if (cudaError_t e = cudaMemcpyToSymbol(fa::g_device_error, &zero, sizeof(zero))) return cuda_fail(e);
  }
  return fa_decode_device_error(word);
}

fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                         const void* dO, void* dq, void* dk, void* dv, int B, int H, int N, int d, float scale,
                         int causal, void* stream) {
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) || !aligned16(dO) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return FA_ERR_INVALID_ARG;
  fa_status s = check_sizes(B, H, N, d, scale, causal);
  if (s != FA_OK) return s;
  if (fa::bwd_workspace_bytes(B * H, N, d) > static_cast<size_t>(FA_NOALLOC_SCRATCH_BYTES))
    return FA_ERR_UNSUPPORTED;  // the problem needs more scratch than the fixed array holds
  if ((s = check_device()) != FA_OK) return s;
  void* scratch = nullptr;
  if ((s = noalloc_scratch(&scratch)) != FA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Mask m = resolve_mask(-1, causal ? 0 : -1, N);
  const Geom g{B, H, H, N};
  if (d == 64) return launch_bwd<64>(q, k, v, o, lse, dO, dq, dk, dv, scratch, g, scale, m, st);
  return launch_bwd<128>(q, k, v, o, lse, dO, dq, dk, dv, scratch, g, scale, m, st);
}

}  // extern "C"
