// fa_bwd.cuh - attention backward for sm_100a: dO.O row-dot, the main
// recompute kernel (TMA + tcgen05 + TMEM), and the dQ fp32 -> bf16 convert.
//
// Method: "FlashAttention原理：从原始Attention到FlashAttention"
// (blog.csdn.net/qq_43527718), section 二 "做法" and section 二.5: the forward
// stores only the softmax normalisation (lse) and the backward recomputes the
// attention matrix tile by tile on chip instead of reading it from HBM. The
// gradient formulas are the calculus of the forward:
//   P = exp(scale*Q K^T - lse),  dV = P^T dO,  dP = dO V^T,
//   D_i = rowsum(dO_i * O_i),    dS = P * (dP - D),
//   dQ = scale * dS K,           dK = scale * dS^T Q.
//
// Main kernel: one CTA per (batch*K/V head, 128-key tile j); it loops over
// 128-query tiles i (causal: only i >= j, the masked upper triangle is
// skipped) of every query head reading that K/V head, and keeps dK_j, dV_j
// accumulating in TMEM. Everything is computed transposed (keys on TMEM
// lanes) so P^T and dS^T can feed the dV/dK MMAs straight from TMEM:
//   S^T  = K_j Q_i^T        (SS, M=128 keys, N=128 queries)  -> TMEM
//   dP^T = V_j dO_i^T       (SS)                             -> TMEM
//   P^T  = 2^(lambda*S^T - lse2),  dS^T = scale * P^T * (dP^T - D)   (registers)
//   dV  += P^T dO_i         (TS: A = P^T bf16 in TMEM)
//   dK  += dS^T Q_i         (TS: A = dS^T bf16 in TMEM)
//   dQ_i^T = K_j^T dS^T     (SS: A = K_j read MN-major, B = dS from smem)
//   dQ_i^T is drained from TMEM by a warpgroup that stages it in shared
//   memory and adds it into the fp32 dQ accumulator with TMA reduce-adds.
// All five products are N = 128 (or N = D) instructions; the TMEM regions are
// single-buffered and their reuse is ordered as described at the kernel.
//
// Roles (512 threads): warp 0 TMA producer (Q with its lse2 and D rows, dO),
// warps 1 to 3 MMA issuers, warps 4-7 the dQ drain warpgroup (thread =
// head-dim row of dQ^T), warps 8-11 and 12-15 two elementwise warpgroups
// (thread = key row) that take query columns 0-63 and 64-127 of every tile.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include "fa_ptx.cuh"

namespace fa {

// The dV MMAs of an iteration wait for its dP^T MMAs to finish (1) or go to
// the tensor pipe as soon as P is ready (0).
#ifndef FA_BWD_DP_FIRST
#define FA_BWD_DP_FIRST 1
#endif
constexpr bool kDpFirst = FA_BWD_DP_FIRST != 0;
// Y commits the release of Q(it)'s ring stage after dQ^T(it) is issued (1),
// so dQ^T, which the dQ drain waits for, is not queued behind the commit; or
// between dK(it) and dQ^T(it) (0).
#ifndef FA_BWD_Q_RELEASE_LATE
#define FA_BWD_Q_RELEASE_LATE 1
#endif

inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Row stride (elements) of the per-row statistics in the workspace: N rounded
// up to a multiple of 4 so each row starts on a 16-byte boundary (TMA rule).
inline int stat_stride(int N) { return (N + 3) & ~3; }

// Workspace: [dQ accumulator fp32 BH*N*d][lse2 fp32 BH*Np][D fp32 BH*Np],
// each piece starting on a 256-byte boundary (Np = stat_stride(N)).
inline size_t bwd_workspace_bytes(int BH, int N, int d) {
  const size_t rows = static_cast<size_t>(BH) * N;
  const size_t srows = static_cast<size_t>(BH) * stat_stride(N);
  return align256(rows * d * sizeof(float)) + 2 * align256(srows * sizeof(float));
}

// Grouped-query attention (Hkv < H) appends fp32 dK and dV accumulators
// [2][B*Hkv*N*d], for when a K/V head's query heads are split across CTAs.
inline size_t bwd_kv_acc_bytes(int B, int Hkv, int N, int d) {
  return align256(static_cast<size_t>(B) * Hkv * N * d * sizeof(float));
}
inline size_t bwd_gqa_workspace_bytes(int B, int H, int Hkv, int N, int d) {
  return bwd_workspace_bytes(B * H, N, d) + (Hkv < H ? 2 * bwd_kv_acc_bytes(B, Hkv, N, d) : 0);
}

// Packed variable-length batches keep the per-row statistics per head in a
// row of varlen_stat_stride(T, B) floats, sequence b starting at the 4-aligned
// position round_up(cu[b], 4) + 4 b (a TMA load must start on a 16-byte
// boundary). The +4b keeps sequences apart however their starts round; the
// positions between one sequence's end and the next start, and the tail after
// the last, hold zeros, so a tile that reaches past its sequence reads finite
// values.
inline int varlen_stat_stride(int T, int B) { return (T + 4 * B + 4 + 3) & ~3; }
__host__ __device__ __forceinline__ int varlen_stat_start(int s0, int b) { return ((s0 + 3) & ~3) + 4 * b; }
inline size_t bwd_varlen_workspace_bytes(int B, int T, int H, int Hkv, int d) {
  const size_t stats = static_cast<size_t>(H) * varlen_stat_stride(T, B) * sizeof(float);
  return align256(static_cast<size_t>(T) * H * d * sizeof(float)) + 2 * align256(stats) +
         (Hkv < H ? 2 * bwd_kv_acc_bytes(1, Hkv, T, d) : 0);
}

// ------------------------------------------------- D = rowsum(dO*O), lse2
// For every query row: D = sum_k dO_k * O_k, lse2 = lse * log2(e) (the
// forward's natural-log normaliser moved to base 2 for the exp2 recompute),
// both written with the padded row stride Np; and the row of the fp32 dQ
// accumulator is zeroed (same rows, same pass). kv_n4 float4s at kv_acc (the
// split grouped-query dK/dV accumulators, or none) are zeroed too.
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_dot_kernel(const __nv_bfloat16* __restrict__ o,
                                                         const __nv_bfloat16* __restrict__ dO,
                                                         const float* __restrict__ lse, float* __restrict__ lse2,
                                                         float* __restrict__ dsum, float* __restrict__ dq_acc,
                                                         long long rows, int N, int Np, float* __restrict__ kv_acc,
                                                         long long kv_n4) {
  constexpr int TPR = D / 8;  // threads per row, 16 bytes of each tensor per thread
  const long long tid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int part = static_cast<int>(tid % TPR);
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x / TPR;
  // A warp covers 32 / TPR consecutive rows and steps through them together,
  // so every lane runs the same iterations (the shuffles need the full warp);
  // lanes whose row is past the end take part with zeros and store nothing.
  const int lane = threadIdx.x & 31;
  for (long long row0 = (tid - lane) / TPR; row0 < rows; row0 += stride) {
    const long long row = row0 + lane / TPR;
    const bool live = row < rows;
    const size_t off = static_cast<size_t>(live ? row : 0) * D + part * 8;
    const uint4 a = live ? __ldg(reinterpret_cast<const uint4*>(o + off)) : make_uint4(0u, 0u, 0u, 0u);
    const uint4 g = live ? __ldg(reinterpret_cast<const uint4*>(dO + off)) : make_uint4(0u, 0u, 0u, 0u);
    const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&g);
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 af = __bfloat1622float2(a2[e]);
      const float2 gf = __bfloat1622float2(g2[e]);
      s = fmaf(af.x, gf.x, s);
      s = fmaf(af.y, gf.y, s);
    }
#pragma unroll
    for (int w = TPR / 2; w >= 1; w >>= 1) s += __shfl_xor_sync(0xffffffffu, s, w);
    if (!live) continue;
    if (part == 0) {
      const long long bh = row / N, qi = row - bh * N;
      const size_t so = static_cast<size_t>(bh) * Np + qi;
      dsum[so] = s;
      lse2[so] = __ldg(lse + row) * 1.4426950408889634f;
    }
    float4* z = reinterpret_cast<float4*>(dq_acc + off);
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  const long long all = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = tid; i < kv_n4; i += all)
    reinterpret_cast<float4*>(kv_acc)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// The same for a packed variable-length batch ([T, H, D] tensors, lse [H, T]),
// one sequence per blockIdx.y step: row (token i of sequence b, head h) puts
// D and lse2 at position varlen_stat_start(s0, b) + i of head h's statistics
// row, zeroes its dQ accumulator row, and the gap up to the next sequence's
// start (the whole tail, after the last sequence) is zeroed. kv_n4 float4s at
// kv_acc are zeroed by the blocks of blockIdx.y == 0.
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_dot_varlen_kernel(
    const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dO, const float* __restrict__ lse,
    float* __restrict__ lse2, float* __restrict__ dsum, float* __restrict__ dq_acc, const int* __restrict__ cu,
    int B, int T, int H, int max_len, int Sp, float* __restrict__ kv_acc, long long kv_n4) {
  constexpr int TPR = D / 8;
  const int tid = static_cast<int>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int part = tid % TPR;
  const int stride = static_cast<int>(gridDim.x) * blockDim.x / TPR;
  const int lane = threadIdx.x & 31;
  for (int b = blockIdx.y; b < B; b += gridDim.y) {
    int s0, L;
    seq_range(cu, b, T, max_len, s0, L);
    const int P = varlen_stat_start(s0, b);
    const int P_end = (b == B - 1) ? Sp : varlen_stat_start(s0 + L, b + 1);
    const int rows = L * H;
    // Warp-uniform row loop, as in fa_bwd_dot_kernel.
    for (int r0 = (tid - lane) / TPR; r0 < rows; r0 += stride) {
      const int r = r0 + lane / TPR;
      const bool live = r < rows;
      const int i = (live ? r : 0) / H, h = (live ? r : 0) - i * H;
      const size_t off = (static_cast<size_t>(s0 + i) * H + h) * D + part * 8;
      const uint4 a = live ? __ldg(reinterpret_cast<const uint4*>(o + off)) : make_uint4(0u, 0u, 0u, 0u);
      const uint4 g = live ? __ldg(reinterpret_cast<const uint4*>(dO + off)) : make_uint4(0u, 0u, 0u, 0u);
      const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
      const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&g);
      float sum = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 af = __bfloat1622float2(a2[e]);
        const float2 gf = __bfloat1622float2(g2[e]);
        sum = fmaf(af.x, gf.x, sum);
        sum = fmaf(af.y, gf.y, sum);
      }
#pragma unroll
      for (int w = TPR / 2; w >= 1; w >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, w);
      if (!live) continue;
      if (part == 0) {
        const size_t so = static_cast<size_t>(h) * Sp + P + i;
        dsum[so] = sum;
        lse2[so] = __ldg(lse + static_cast<size_t>(h) * T + s0 + i) * 1.4426950408889634f;
      }
      float4* z = reinterpret_cast<float4*>(dq_acc + off);
      z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
      z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    // Zero the statistics between this sequence's end and the next start.
    const int gap = max(P_end - (P + L), 0);
    for (int r = tid; r < gap * H; r += static_cast<int>(gridDim.x) * blockDim.x) {
      const int h = r / gap;
      const size_t so = static_cast<size_t>(h) * Sp + P + L + (r - h * gap);
      dsum[so] = 0.f;
      lse2[so] = 0.f;
    }
  }
  if (blockIdx.y == 0) {
    const long long all = static_cast<long long>(gridDim.x) * blockDim.x;
    for (long long i = tid; i < kv_n4; i += all)
      reinterpret_cast<float4*>(kv_acc)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// --------------------------------------------------------- dQ fp32 -> bf16
__global__ void __launch_bounds__(256) fa_bwd_dq_convert_kernel(const float* __restrict__ acc,
                                                                __nv_bfloat16* __restrict__ dq, long long n8) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8; i += stride) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(acc) + 2 * i);
    const float4 b = __ldg(reinterpret_cast<const float4*>(acc) + 2 * i + 1);
    uint4 w;
    w.x = pack_bf16(a.x, a.y);
    w.y = pack_bf16(a.z, a.w);
    w.z = pack_bf16(b.x, b.y);
    w.w = pack_bf16(b.z, b.w);
    reinterpret_cast<uint4*>(dq)[i] = w;
  }
}

// ------------------------------------------------------------------ main kernel
struct BwdParams {
  int BH;         // batch * K/V heads * n_split: one CTA per (unit, 128-key tile)
  int H;          // query heads
  int Hkv;        // K/V heads; query heads [g*H/Hkv, (g+1)*H/Hkv) share K/V head g
  int n_split;    // CTAs that share one K/V head's query heads (divides H/Hkv); > 1: dK, dV add into fp32
  int wl, wr;     // band mask only: key j visible to query i iff i - wl <= j <= i + wr (0 <= wl, wr <= N)
  int sched_groups;  // causal launch order: number of unit groups (1 <= sched_groups <= BH)
  const int* cu_seqlens;  // packed variable length ([T, heads, D] tensors): [B + 1] prefix sums; else nullptr
  int T;                  // packed rows (variable length only); N is then the longest length
  int N;
  int n_kv;          // ceil(N / 128)
  float scale;       // softmax scale
  float scale_log2;  // scale * log2(e)
  // Rows of a ragged last key tile that the TMA store cannot clip (packed
  // layout) are written by the threads themselves, here:
  void* dk;          // bf16 [.., D] (n_split == 1)
  void* dv;
  float* dk_acc;     // fp32 [.., D], zeroed (n_split > 1)
  float* dv_acc;
};

// Shared memory of the main kernel (bytes). A tile is 128 rows x D bf16, kept
// as D/64 column chunks of [128 rows][128 B] with the 128-byte swizzle.
template <int D>
struct BwdLayout {
  static constexpr int kChunk = 128 * 128;              // one 64-column chunk of a 128-row tile
  static constexpr int kTile = 128 * D * 2;
  static constexpr int kQS = (D == 128) ? 2 : 3;        // Q (+ lse2, D statistics) ring
  static constexpr int kDOS = (D == 128) ? 1 : 2;       // dO ring
  static constexpr int kK = 0;
  static constexpr int kV = kTile;
  static constexpr int kQ = 2 * kTile;
  static constexpr int kDO = kQ + kQS * kTile;
  // dS tile as the MN-major operand of dQ^T: [2 query groups of 64][128 keys][128 B].
  static constexpr int kDS = kDO + kDOS * kTile;
  static constexpr int kDSTile = 128 * 128 * 2;
  // Two fp32 staging buffers for dQ^T, 32 queries x D each: one is written
  // while the TMA engine still reads the other.
  static constexpr int kStgHalf = 32 * D * 4;
  static constexpr int kStg = kDS + kDSTile;
  static constexpr int kStat = kStg + 2 * kStgHalf;     // [kQS] x {lse2[128], D[128]} fp32
  static constexpr int kBar = kStat + kQS * 1024;
  static constexpr int kBytes = kBar + 256;
  // The kernel checks that the dynamic shared memory base is 1 KB aligned
  // (it is: the window starts on a 1 KB boundary) instead of reserving slack.
  static constexpr int kAlloc = kBytes;
  static_assert(kAlloc <= 227 * 1024, "shared memory budget");
  // Epilogue staging of dK/dV, one slot per elementwise warp (8), from offset
  // 0: K, V and the Q ring are free by then.
  static constexpr int kEpiBf16 = 32 * D * 2;
  static constexpr int kEpiF32 = 32 * D * 4;
  static_assert(8 * kEpiF32 <= kDO, "epilogue staging must fit in K, V and the Q ring");
};

// Roles, one warpgroup each: warps 0-3 control (warp 0 TMA producer, warps 1-3
// MMA issuers X, Y, Z; warp 1 also owns TMEM), 4-7 dQ drain, 8-11 and 12-15
// elementwise (query columns 0-63 and 64-127 of every tile). Launched at 128
// registers per thread (512 x 128 = the 64K register file; each SM
// sub-partition holds one warp of every warpgroup); the groups then move to
// 56 / 152 / 152 / 152, which sums to the same 512 per slot.
constexpr int kBwdThreads = 512;
constexpr int kRegCtl = 56, kRegDrain = 152, kRegElem = 152;
static_assert(kRegCtl + kRegDrain + 2 * kRegElem == 512, "register split must equal the launch budget");

__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Main backward kernel: one CTA per (batch*K/V head*share, 128-key tile j),
// iterating over the 128-query tiles that see a key of the tile.
//
// TMEM (512 columns): S^T [0,128) with P^T (bf16) written over it, dP^T
// [128,256) with dS^T (bf16) written over it and then dQ^T over both, dV at
// 256, dK at 256 + D. Every region is single-buffered; reuse is ordered
// either by one issuing thread (tcgen05.mma from one thread execute in issue
// order) or by a barrier:
//   X: dV(i) [after P^T(i)], then S^T(i+1) over S^T/P^T(i).
//   Y: dK(i) [after dS^T(i)], then dQ^T(i) over dP^T/dS^T(i).
//   Z: dP^T(i+1) over dQ^T(i), after the drain has copied dQ^T(i) out.
// The elementwise groups turn S^T(i) into P^T(i) while Y and Z work on
// iteration i-1's dK, dQ^T and the next dP^T, and turn dP^T(i) into dS^T(i)
// while X computes dV(i) and S^T(i+1).
template <int D, int MASK>
__global__ void __launch_bounds__(kBwdThreads, 1)
    fa_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                  const __grid_constant__ CUtensorMap tm_dq, const __grid_constant__ CUtensorMap tm_lse2,
                  const __grid_constant__ CUtensorMap tm_dsum, const __grid_constant__ CUtensorMap tm_dk,
                  const __grid_constant__ CUtensorMap tm_dv, const BwdParams p) {
  using L = BwdLayout<D>;
  constexpr int QS = L::kQS;
  constexpr int DOS = L::kDOS;
  constexpr int KCH = D / 64;

  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_u32(smem) & 1023u) != 0u) {  // uniform over the CTA: nothing started yet
    if (threadIdx.x == 0) atomicOr(&g_device_error, kDevErrSmemAlign);
    return;
  }

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* kv_full = bars;
  uint64_t* q_full = kv_full + 1;       // [QS] Q tile + statistics landed
  uint64_t* q_empty = q_full + QS;      // [QS] S^T (X) and dK (Y) done reading
  uint64_t* do_full = q_empty + QS;     // [DOS]
  uint64_t* do_empty = do_full + DOS;   // [DOS] dP^T (Z) and dV (X) done reading
  uint64_t* s_full = do_empty + DOS;
  uint64_t* p_full = s_full + 1;
  uint64_t* dp_full = p_full + 1;
  uint64_t* ds_full = dp_full + 1;
  uint64_t* dq_full = ds_full + 1;
  uint64_t* dq_empty = dq_full + 1;
  uint64_t* acc_full = dq_empty + 1;
  uint64_t* mma_done = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  static_assert((1 + 2 * QS + 2 * DOS + 8) * 8 + 8 <= 256, "barrier region");

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Causal: key tile 0 sees every query tile, so low j first (heaviest),
  // within sched_groups groups of units, each small enough that its Q, dO and
  // dQ accumulator stay in L2 (grouped_order). Otherwise unit-major.
  int j, unit;
  if (MASK == kMaskCausal) {
    grouped_order(static_cast<int>(blockIdx.x), p.BH, p.sched_groups, p.n_kv, j, unit);
  } else {
    unit = static_cast<int>(blockIdx.x) / p.n_kv;
    j = static_cast<int>(blockIdx.x) % p.n_kv;
  }
  // The CTA walks every query tile of its share of the query heads that read
  // K/V head bkv (the one head, for multi-head attention): dK and dV
  // accumulate on chip over that share, and across the n_split shares in
  // fp32 global memory.
  const int bkv = unit / p.n_split;  // batch * Hkv + K/V head
  // This CTA's sequence: length N, first row s0 in the maps' row dimension.
  // Fixed-length maps index batch*head, packed ones the head alone.
  const bool packed = p.cu_seqlens != nullptr;
  int N = p.N, s0 = 0;
  if (packed) seq_range(p.cu_seqlens, bkv / p.Hkv, p.T, p.N, s0, N);
  if (j * 128 >= N) return;  // past the end of a shorter sequence: the whole CTA leaves
  const int kvh = packed ? bkv % p.Hkv : bkv;  // K/V head coordinate of the maps
  // First position of this sequence in the per-row statistics (4-aligned).
  const int stat0 = packed ? varlen_stat_start(s0, bkv / p.Hkv) : 0;
  const int group = p.H / p.Hkv / p.n_split;   // query heads of this CTA
  const int qh0 = (packed ? 0 : (bkv / p.Hkv) * p.H) + (bkv % p.Hkv) * (p.H / p.Hkv) + (unit % p.n_split) * group;
  const int n_q = (N + 127) / 128;
  // 128-query tiles [i_start, i_end) that see a key of this tile; never
  // empty, since key 128*j < N sees itself.
  int i_start = 0, i_end = n_q;
  if (MASK == kMaskCausal) i_start = j;
  if (MASK == kMaskBand) {
    i_start = max(0, j * 128 - p.wr) / 128;
    i_end = min(n_q, min(j * 128 + 127 + p.wl, N - 1) / 128 + 1);
  }
  const int n_iq = i_end - i_start;  // query tiles per head
  const int n_it = group * n_iq;
  auto q_start = [&](int it) { return (i_start + it % n_iq) * 128; };
  auto q_head = [&](int it) { return qh0 + it / n_iq; };

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < QS; ++s) {
      mbar_init(q_full + s, 1);
      mbar_init(q_empty + s, 2);
    }
    for (int s = 0; s < DOS; ++s) {
      mbar_init(do_full + s, 1);
      mbar_init(do_empty + s, 2);
    }
    mbar_init(s_full, 1);
    mbar_init(p_full, 8);    // one arrival per elementwise warp
    mbar_init(dp_full, 1);
    mbar_init(ds_full, 8);
    mbar_init(dq_full, 1);
    mbar_init(dq_empty, 4);  // one arrival per drain warp
    mbar_init(acc_full, 2);  // last dV (X) and last dK + dQ^T (Y)
    mbar_init(mma_done, 3);  // one per MMA issuer
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int wg = warp >> 2;
  constexpr uint32_t t_dp = 128, t_dv = 256, t_dk = 256 + D;
  constexpr uint32_t kQTx = L::kTile + 1024;  // Q tile + lse2[128] + D[128]

  if (wg == 0) setmaxnreg_dec<kRegCtl>();
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // Loads in the order they are needed: Q(i) (needed by S^T(i)), then
    // dO(i) (needed by dP^T(i), which comes later).
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      prefetch_tmap(&tm_do);
      prefetch_tmap(&tm_dq);
      prefetch_tmap(&tm_lse2);
      prefetch_tmap(&tm_dsum);
      mbar_arrive_expect_tx(kv_full, 2 * L::kTile);
      for (int c = 0; c < KCH; ++c) {
        tma_load_3d(smem + L::kK + c * L::kChunk, &tm_k, kv_full, c * 64, s0 + j * 128, kvh);
        tma_load_3d(smem + L::kV + c * L::kChunk, &tm_v, kv_full, c * 64, s0 + j * 128, kvh);
      }
      int q_issued = 0, do_issued = 0;
      for (int it = 0; it < n_it; ++it) {
        const int q0 = q_start(it), bhq = q_head(it);
        const int s = it % QS;
        if (it >= QS && !wait_parity(q_empty + s, (it / QS - 1) & 1, abort_flag)) break;
        uint8_t* st = smem + L::kStat + s * 1024;
        mbar_arrive_expect_tx(q_full + s, kQTx);
        for (int c = 0; c < KCH; ++c)
          tma_load_3d(smem + L::kQ + s * L::kTile + c * L::kChunk, &tm_q, q_full + s, c * 64, s0 + q0, bhq);
        tma_load_2d(st, &tm_lse2, q_full + s, stat0 + q0, bhq);
        tma_load_2d(st + 512, &tm_dsum, q_full + s, stat0 + q0, bhq);
        q_issued = it + 1;
        const int t = it % DOS;
        if (it >= DOS && !wait_parity(do_empty + t, (it / DOS - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(do_full + t, L::kTile);
        for (int c = 0; c < KCH; ++c)
          tma_load_3d(smem + L::kDO + t * L::kTile + c * L::kChunk, &tm_do, do_full + t, c * 64, s0 + q0, bhq);
        do_issued = it + 1;
      }
      // Every copy this thread started must land before the CTA exits.
      wait_parity_drain(kv_full, 0);
      for (int it = max(0, q_issued - QS); it < q_issued; ++it) wait_parity_drain(q_full + it % QS, (it / QS) & 1);
      for (int it = max(0, do_issued - DOS); it < do_issued; ++it)
        wait_parity_drain(do_full + it % DOS, (it / DOS) & 1);
    }
  } else if (warp >= 1 && warp <= 3) {
    // ------------------------------------------------------- MMA issuers
    // Three threads share the 40 instructions of an iteration, so that
    // products that do not depend on each other are in the tensor pipe
    // together: X (warp 1) dV and S^T, Y (warp 2) dK and dQ^T, Z (warp 3) dP^T.
    if (lane == 0) {
      constexpr uint32_t kIdST = idesc_bf16(128, 128, 0, 0);  // S^T, dP^T: K-major A and B
      constexpr uint32_t kIdAcc = idesc_bf16(128, D, 0, 1);   // dV, dK: A in TMEM, B MN-major
      constexpr uint32_t kIdDQ = idesc_bf16(D, 128, 1, 1);    // dQ^T: A, B MN-major
      const uint32_t k_addr = smem_u32(smem + L::kK);
      const uint32_t v_addr = smem_u32(smem + L::kV);
      const uint32_t q_addr = smem_u32(smem + L::kQ);
      const uint32_t do_addr = smem_u32(smem + L::kDO);
      const uint32_t ds_addr = smem_u32(smem + L::kDS);

      // X^T = A_j Y^T: A_j a 128-key K/V tile, Y a 128-query Q/dO tile, both K-major.
      auto issue_t = [&](uint32_t d_col, uint32_t a_base, uint32_t b_base) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * L::kChunk + (kk & 3) * 32;
          mma_ss(tmem + d_col, sdesc_sw128(a_base + off, 16, 1024), sdesc_sw128(b_base + off, 16, 1024), kIdST,
                 kk > 0);
        }
      };
      // acc += X^T * Y: X^T the bf16 [128 keys][128 queries] in TMEM, written
      // by the elementwise groups at columns a_col + 64 g + [0, 32) for query
      // group g; Y a 128-query tile read MN-major (D contiguous).
      auto issue_acc = [&](uint32_t d_col, uint32_t a_col, uint32_t b_base, bool acc) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tmem + d_col, tmem + a_col + 64 * (kk >> 2) + 8 * (kk & 3),
                 sdesc_sw128(b_base + kk * 2048, L::kChunk, 1024), kIdAcc, (acc || kk > 0) ? 1u : 0u);
      };
      // dQ^T = K_j^T dS^T: K read MN-major (D contiguous), dS from the
      // shared-memory tile, MN-major (queries contiguous).
      auto issue_dq = [&]() {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tmem + t_dp, sdesc_sw128(k_addr + kk * 2048, L::kChunk, 1024),
                 sdesc_sw128(ds_addr + kk * 2048, 128 * 128, 1024), kIdDQ, kk > 0);
      };

      const int role = warp - 1;  // 0 X, 1 Y, 2 Z
      bool ok = wait_parity(kv_full, 0, abort_flag);
      if (role == 0) {
        if (ok && (ok = wait_parity(q_full, 0, abort_flag))) {
          tc_fence_after();
          issue_t(0, k_addr, q_addr);
          mma_commit(s_full);
          mma_commit(q_empty);
        }
        for (int it = 0; ok && it < n_it; ++it) {
          const int t = it % DOS;
          // dV(it) reads dO(it): nothing else X waits for implies it landed.
          if (!(ok = wait_parity(do_full + t, (it / DOS) & 1, abort_flag))) break;
          if (!(ok = wait_parity(p_full, it & 1, abort_flag))) break;
          // dP^T(it) is on the critical chain (dP^T -> dS phase -> dK, dQ^T ->
          // drain -> next dP^T) and dV(it) is not, so dV waits until dP^T(it)
          // has had the tensor pipe. With one dO stage, dP^T(it+1) needs
          // dO(it+1), whose load needs dV(it) done, so dp_full cannot be two
          // phases ahead of this wait.
          if (kDpFirst && DOS == 1 && !(ok = wait_parity(dp_full, it & 1, abort_flag))) break;
          tc_fence_after();
          issue_acc(t_dv, 0, do_addr + t * L::kTile, it > 0);
          mma_commit(do_empty + t);
          if (it + 1 < n_it) {
            const int ns = (it + 1) % QS;
            if (!(ok = wait_parity(q_full + ns, ((it + 1) / QS) & 1, abort_flag))) break;
            tc_fence_after();
            issue_t(0, k_addr, q_addr + ns * L::kTile);  // over P^T(it): after dV(it), same thread
            mma_commit(s_full);
            mma_commit(q_empty + ns);
          }
        }
      } else if (role == 1) {
        for (int it = 0; ok && it < n_it; ++it) {
          const int s = it % QS;
          // dS^T(it) implies S^T(it) and so Q(it); the Q wait is explicit anyway.
          if (!(ok = wait_parity(q_full + s, (it / QS) & 1, abort_flag))) break;
          if (!(ok = wait_parity(ds_full, it & 1, abort_flag))) break;
          tc_fence_after();
          issue_acc(t_dk, t_dp, q_addr + s * L::kTile, it > 0);
          if (!FA_BWD_Q_RELEASE_LATE) mma_commit(q_empty + s);
          issue_dq();  // over dS^T(it): after dK(it), same thread
          mma_commit(dq_full);
          if (FA_BWD_Q_RELEASE_LATE) mma_commit(q_empty + s);
        }
      } else {
        if (ok && (ok = wait_parity(do_full, 0, abort_flag))) {
          tc_fence_after();
          issue_t(t_dp, v_addr, do_addr);
          mma_commit(dp_full);
          mma_commit(do_empty);
        }
        for (int it = 0; ok && it + 1 < n_it; ++it) {
          const int nt = (it + 1) % DOS;
          if (!(ok = wait_parity(dq_empty, it & 1, abort_flag))) break;
          if (!(ok = wait_parity(do_full + nt, ((it + 1) / DOS) & 1, abort_flag))) break;
          tc_fence_after();
          issue_t(t_dp, v_addr, do_addr + nt * L::kTile);
          mma_commit(dp_full);
          mma_commit(do_empty + nt);
        }
      }
      if (ok && role < 2) mma_commit(acc_full);
      // Let every MMA the issuers started finish before TMEM is freed.
      mma_commit(mma_done);
      wait_parity_drain(mma_done, 0);
    }
  } else if (wg >= 2) {
    // ---------------------------------------- elementwise (thread = key row)
    // Group e takes query columns [64e, 64e + 64) of every tile.
    setmaxnreg_inc<kRegElem>();
    const int e = wg - 2;
    const int quarter = warp & 3;
    const int k = quarter * 32 + lane;
    const int kj = j * 128 + k;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const float lam = p.scale_log2;
    const float scale = p.scale;
    const uint32_t tS = tmem + lane_off + 64 * e;
    const uint32_t tP = tmem + lane_off + t_dp + 64 * e;
    uint8_t* ds_row = smem + L::kDS + e * (128 * 128) + k * 128;
    bool ok = true;
    for (int it = 0; it < n_it; ++it) {
      const int s = it % QS;
      const int qe = q_start(it) + 64 * e;  // first query of this group's columns
      ok = __all_sync(0xffffffffu, wait_parity(q_full + s, (it / QS) & 1, abort_flag) &&
                                       wait_parity(s_full, it & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      const float4* lse2 = reinterpret_cast<const float4*>(smem + L::kStat + s * 1024) + 16 * e;
      const float4* dd = reinterpret_cast<const float4*>(smem + L::kStat + s * 1024 + 512) + 16 * e;
      const bool edge = (qe + 64 > N) || (j * 128 + 128 > N) || (MASK == kMaskCausal && j * 128 + 127 > qe) ||
                        (MASK == kMaskBand && (j * 128 + 127 > qe + p.wr || j * 128 < qe + 63 - p.wl));
      float pr[64];
      {
        uint32_t sv[64];
        tmem_ld64(tS, sv);
        tmem_wait_ld();
#pragma unroll
        for (int c4 = 0; c4 < 16; ++c4) {
          const float4 l4 = lse2[c4];
          // Packed f32x2: scale and subtract for two queries per instruction.
          const float2 lam2 = make_float2(lam, lam);
          const float2 x01 = ffma2(make_float2(__uint_as_float(sv[4 * c4 + 0]), __uint_as_float(sv[4 * c4 + 1])), lam2,
                                   make_float2(-l4.x, -l4.y));
          const float2 x23 = ffma2(make_float2(__uint_as_float(sv[4 * c4 + 2]), __uint_as_float(sv[4 * c4 + 3])), lam2,
                                   make_float2(-l4.z, -l4.w));
          pr[4 * c4 + 0] = ex2(x01.x);
          pr[4 * c4 + 1] = ex2(x01.y);
          pr[4 * c4 + 2] = ex2(x23.x);
          pr[4 * c4 + 3] = ex2(x23.y);
        }
      }
      if (edge) {
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const int qi = qe + c;
          const bool vis = (qi < N) && (kj < N) && (MASK != kMaskCausal || kj <= qi) &&
                           (MASK != kMaskBand || (kj >= qi - p.wl && kj <= qi + p.wr));
          if (!vis) pr[c] = 0.f;
        }
      }
      {
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) pk[c] = pack_bf16(pr[2 * c], pr[2 * c + 1]);
        tmem_st32(tS, pk);  // P^T over this thread's own S^T columns
      }
      // dS = (scale P) (dP - D): the scale is applied here, off the dS
      // phase, which is on the iteration's critical path.
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const float2 ps = fmul2(make_float2(pr[2 * c], pr[2 * c + 1]), make_float2(scale, scale));
        pr[2 * c] = ps.x;
        pr[2 * c + 1] = ps.y;
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);

      // The dS tile was last read by dQ^T(it - 1), which finished before the
      // drain released dQ^T's TMEM and so before dP^T(it) was issued.
      ok = __all_sync(0xffffffffu, wait_parity(dp_full, it & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      // Both halves of this group's dP^T columns in one TMEM round trip.
      uint32_t dpa[64];
      tmem_ld32(tP + 0, dpa);
      tmem_ld32(tP + 32, dpa + 32);
      tmem_wait_ld();
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t* dp = dpa + 32 * h;
        uint32_t pk[16];
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4) {
          const float4 d4 = dd[8 * h + c4];
          const int q = 32 * h + 4 * c4;
          // Packed f32x2: one sub and one mul per pair of queries.
          const float2 g01 = fmul2(make_float2(pr[q + 0], pr[q + 1]),
                                   fsub2(make_float2(__uint_as_float(dp[4 * c4 + 0]), __uint_as_float(dp[4 * c4 + 1])),
                                         make_float2(d4.x, d4.y)));
          const float2 g23 = fmul2(make_float2(pr[q + 2], pr[q + 3]),
                                   fsub2(make_float2(__uint_as_float(dp[4 * c4 + 2]), __uint_as_float(dp[4 * c4 + 3])),
                                         make_float2(d4.z, d4.w)));
          pk[2 * c4] = pack_bf16(g01.x, g01.y);
          pk[2 * c4 + 1] = pack_bf16(g23.x, g23.y);
        }
        // dS^T over dP^T columns this thread has already read.
        tmem_st16(tP + 16 * h, pk);
        // Row k of the [128 keys][64 queries] dS group tile, 128-byte
        // swizzle: 16-byte chunk c (queries 8c..8c+7) lives at chunk c ^ (k & 7).
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int chunk = 4 * h + c;
          *reinterpret_cast<uint4*>(ds_row + ((chunk ^ (k & 7)) << 4)) =
              make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        }
      }
      fence_proxy_async_smem();
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(ds_full);
    }
    // ------------------------------ epilogue: group 0 writes dV, group 1 dK
    // Each warp stages its 32 key rows in shared memory (128-byte swizzle)
    // and writes them with TMA: a bf16 store, or, when CTAs share a K/V
    // head's query heads, an fp32 reduce-add into the accumulator. Rows a
    // TMA store cannot clip (past the end of a packed sequence) are written
    // by the threads.
    if (ok) {
      ok = __all_sync(0xffffffffu, wait_parity(acc_full, 0, abort_flag));
      if (ok) {
        tc_fence_after();
        const bool split = p.n_split > 1;
        const int r0 = j * 128 + quarter * 32;  // this warp's first key
        const uint32_t col = e ? t_dk : t_dv;
        const CUtensorMap* tm_out = e ? &tm_dk : &tm_dv;
        if (r0 < N && (!packed || r0 + 32 <= N)) {
          const int slot = e * 4 + quarter;
          uint8_t* stg = smem + slot * (split ? L::kEpiF32 : L::kEpiBf16);
          uint8_t* row = stg + lane * 128;
          const int sw = lane & 7;
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t v[32];
            tmem_ld32(tmem + lane_off + col + 32 * c, v);
            tmem_wait_ld();
            if (split) {
              // fp32 chunk c: [32 rows][32 columns = 128 B]
#pragma unroll
              for (int u = 0; u < 8; ++u)
                *reinterpret_cast<uint4*>(row + c * 4096 + ((u ^ sw) << 4)) =
                    make_uint4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
            } else {
              // bf16 chunk c/2: [32 rows][64 columns = 128 B], units 4(c&1)..+3
#pragma unroll
              for (int x = 0; x < 4; ++x) {
                const int u = 4 * (c & 1) + x;
                *reinterpret_cast<uint4*>(row + (c >> 1) * 4096 + ((u ^ sw) << 4)) =
                    make_uint4(pack_bf16(__uint_as_float(v[8 * x]), __uint_as_float(v[8 * x + 1])),
                               pack_bf16(__uint_as_float(v[8 * x + 2]), __uint_as_float(v[8 * x + 3])),
                               pack_bf16(__uint_as_float(v[8 * x + 4]), __uint_as_float(v[8 * x + 5])),
                               pack_bf16(__uint_as_float(v[8 * x + 6]), __uint_as_float(v[8 * x + 7])));
              }
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (split) {
#pragma unroll
              for (int c = 0; c < D / 32; ++c) tma_reduce_add_3d(tm_out, stg + c * 4096, 32 * c, s0 + r0, kvh);
            } else {
#pragma unroll
              for (int c = 0; c < D / 64; ++c) tma_store_3d(tm_out, stg + c * 4096, 64 * c, s0 + r0, kvh);
            }
            bulk_commit_group();
            bulk_wait_group0();
          }
          __syncwarp();
        } else {
          const bool valid = kj < N;
          const int kv = valid ? kj : 0;
          // dK/dV row of key kj, in units of D elements.
          const size_t orow =
              packed ? static_cast<size_t>(s0 + kv) * p.Hkv + kvh : static_cast<size_t>(bkv) * N + kv;
          __nv_bfloat16* out = static_cast<__nv_bfloat16*>(e ? p.dk : p.dv) + orow * D;
          float* acc = (e ? p.dk_acc : p.dv_acc) + orow * D;
#pragma unroll
          for (int c = 0; c < D; c += 32) {
            uint32_t v[32];
            tmem_ld32(tmem + lane_off + col + c, v);
            tmem_wait_ld();
            if (valid && split) {
#pragma unroll
              for (int x = 0; x < 8; ++x)
                red_add_v4(acc + c + 4 * x, __uint_as_float(v[4 * x]), __uint_as_float(v[4 * x + 1]),
                           __uint_as_float(v[4 * x + 2]), __uint_as_float(v[4 * x + 3]));
            } else if (valid) {
              uint4* dst = reinterpret_cast<uint4*>(out + c);
#pragma unroll
              for (int x = 0; x < 4; ++x)
                dst[x] = make_uint4(pack_bf16(__uint_as_float(v[8 * x]), __uint_as_float(v[8 * x + 1])),
                                    pack_bf16(__uint_as_float(v[8 * x + 2]), __uint_as_float(v[8 * x + 3])),
                                    pack_bf16(__uint_as_float(v[8 * x + 4]), __uint_as_float(v[8 * x + 5])),
                                    pack_bf16(__uint_as_float(v[8 * x + 6]), __uint_as_float(v[8 * x + 7])));
            }
          }
        }
      }
    }
  } else if (wg == 1) {
    // ------------------------------------------------- dQ drain (warps 4-7)
    // dQ_i^T sits in TMEM with the head-dim index on lanes and the 128
    // queries on columns. The drain copies all of it into registers and
    // releases the TMEM at once (the next dP^T waits for that), then stages
    // it 32 queries at a time in two fp32 [32][D] buffers; one TMA reduce-add
    // per buffer adds it into the fp32 accumulator while the warps stage the
    // next 32 queries.
    setmaxnreg_inc<kRegDrain>();
    const int quarter = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    // M = D = 128 uses every lane; M = 64 uses lanes 0-15 of each quarter.
    const int drow = (D == 128) ? quarter * 32 + lane : quarter * 16 + lane;
    const bool holds = (D == 128) || (lane < 16);
    const bool leader = (warp == 4 && lane == 0);
    bool ok = true;
    // Every drain warp runs all 8*n_it named barriers, even after an abort
    // (work is skipped instead), so no warp can be left waiting at one.
    for (int it = 0; it < n_it; ++it) {
      if (ok) ok = __all_sync(0xffffffffu, wait_parity(dq_full, it & 1, abort_flag));
      uint32_t v[128];
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tmem + lane_off + t_dp + 32 * c, v + 32 * c);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(dq_empty);
      }
      const int q0 = q_start(it), bhq = q_head(it);
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        float* stg = reinterpret_cast<float*>(smem + L::kStg + (h & 1) * L::kStgHalf);
        // Groups go out in order: at most one pending means the previous
        // read of this buffer is done.
        if (leader) bulk_wait_group_read1();
        named_bar_sync(1, 128);
        if (ok && holds) {
#pragma unroll
          for (int q = 0; q < 32; ++q) stg[q * D + drow] = __uint_as_float(v[32 * h + q]);
        }
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (leader && ok) {
          tma_reduce_add_3d(&tm_dq, stg, 0, s0 + q0 + 32 * h, bhq);
          bulk_commit_group();
        }
      }
    }
    if (leader) bulk_wait_group0();
  }

  // ------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace fa
