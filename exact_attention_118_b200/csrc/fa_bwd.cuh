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
// 64-query tiles i (causal: only i with a visible query, the masked upper
// triangle is skipped) of every query head reading that K/V head, and keeps
// dK_j, dV_j accumulating in TMEM. Everything is
// computed transposed (keys on TMEM lanes) so P^T and dS^T can feed the dV/dK
// MMAs straight from TMEM:
//   S^T  = K_j Q_i^T        (SS, M=128 keys, N=64 queries)   -> TMEM S[b]
//   dP^T = V_j dO_i^T       (SS)                             -> TMEM dP[b]
//   P^T  = 2^(lambda*S^T - lse2),  dS^T = scale * P^T * (dP^T - D)   (registers)
//   dV  += P^T dO_i         (TS: A = P^T bf16 in TMEM)
//   dK  += dS^T Q_i         (TS: A = dS^T bf16 in TMEM)
//   dQ_i^T = K_j^T dS^T     (SS: A = K_j read MN-major, B = dS from smem)
//   dQ_i^T is drained from TMEM by a warpgroup that stages it in shared
//   memory and adds it into the fp32 dQ accumulator with TMA reduce-adds.
// S and dP are double-buffered (b = iteration & 1) so the tensor core computes
// tile i+1 while an elementwise warpgroup works on tile i; each buffer has its
// own elementwise warpgroup, so the two groups overlap each other's waits.
//
// Roles (512 threads): warp 0 TMA producer (Q, dO, lse2 and D tiles), warps 1
// to 3 MMA issuers, warps 4-7 the dQ drain warpgroup (thread = head-dim row of
// dQ^T), warps 8-11 and 12-15 two elementwise warpgroups (thread = key row)
// that take alternate query tiles.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include "fa_ptx.cuh"

namespace fa {

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
  for (long long row = tid / TPR; row < rows; row += stride) {
    const size_t off = static_cast<size_t>(row) * D + part * 8;
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(o + off));
    const uint4 g = __ldg(reinterpret_cast<const uint4*>(dO + off));
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
  for (int b = blockIdx.y; b < B; b += gridDim.y) {
    int s0, L;
    seq_range(cu, b, T, max_len, s0, L);
    const int P = varlen_stat_start(s0, b);
    const int P_end = (b == B - 1) ? Sp : varlen_stat_start(s0 + L, b + 1);
    const int rows = L * H;
    for (int r = tid / TPR; r < rows; r += stride) {
      const int i = r / H, h = r - i * H;
      const size_t off = (static_cast<size_t>(s0 + i) * H + h) * D + part * 8;
      const uint4 a = __ldg(reinterpret_cast<const uint4*>(o + off));
      const uint4 g = __ldg(reinterpret_cast<const uint4*>(dO + off));
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
  void* dk;       // bf16 [B, Hkv, N, D]      (n_split == 1)
  void* dv;       // bf16 [B, Hkv, N, D]      (n_split == 1)
  float* dk_acc;  // fp32 [B, Hkv, N, D], zeroed (n_split > 1)
  float* dv_acc;  // fp32 [B, Hkv, N, D], zeroed (n_split > 1)
  int BH;         // batch * K/V heads * n_split: one CTA per (unit, 128-key tile)
  int H;          // query heads
  int Hkv;        // K/V heads; query heads [g*H/Hkv, (g+1)*H/Hkv) share K/V head g
  int n_split;    // CTAs that share one K/V head's query heads (divides H/Hkv)
  int wl, wr;     // band mask only: key j visible to query i iff i - wl <= j <= i + wr (0 <= wl, wr <= N)
  int sched_groups;  // causal launch order: number of unit groups (1 <= sched_groups <= BH)
  const int* cu_seqlens;  // packed variable length ([T, heads, D] tensors): [B + 1] prefix sums; else nullptr
  int T;                  // packed rows (variable length only); N is then the longest length
  int N;
  int n_kv;          // ceil(N / 128)
  float scale;       // softmax scale
  float scale_log2;  // scale * log2(e)
};

template <int D>
struct BwdLayout {
  static constexpr int kKV = 128 * D * 2;  // K or V tile: 128 keys
  static constexpr int kQT = 64 * D * 2;   // Q or dO tile: 64 queries
  static constexpr int kStages = (D == 128) ? 3 : 4;  // Q/dO/lse2/D ring depth
  static constexpr int kDSTile = 128 * 64 * 2;
  static constexpr int kK = 0;
  static constexpr int kV = kKV;
  static constexpr int kQ = 2 * kKV;
  static constexpr int kDO = kQ + kStages * kQT;
  // [2] dS tiles [128 keys][64 queries].
  static constexpr int kDS = kDO + kStages * kQT;
  static constexpr int kStat = kDS + 2 * kDSTile;  // [kStages] x {lse2[64], D[64]}
  // [2] fp32 staging halves for dQ_i (32 queries x D each), so one half is
  // written while the TMA engine still reads the other.
  static constexpr int kStgHalf = 32 * D * 4;
  static constexpr int kStg = (kStat + kStages * 512 + 1023) & ~1023;
  static constexpr int kBar = kStg + 2 * kStgHalf;
  static constexpr int kBytes = kBar + 256;
  // The kernel checks that the dynamic shared memory base is 1 KB aligned
  // (it is: the window starts on a 1 KB boundary) instead of reserving slack.
  static constexpr int kAlloc = kBytes;
  static_assert(kAlloc <= 227 * 1024, "shared memory budget");
};

// Roles, one warpgroup each: warps 0-3 control (warp 0 TMA producer, warps 1-3
// MMA issuers, warp 1 also TMEM owner), 4-7 dQ drain, 8-11 elementwise
// (even iterations, TMEM buffer 0), 12-15 elementwise (odd iterations, buffer
// 1). Launched at 128 registers per thread (512 x 128 = the 64K register
// file; each SM sub-partition holds one warp of every warpgroup); the groups
// then move to 56 / 104 / 176 / 176, which sums to the same 512 per slot.
constexpr int kBwdThreads = 512;
constexpr int kRegCtl = 56, kRegDrain = 104, kRegElem = 176;
static_assert(kRegCtl + kRegDrain + 2 * kRegElem == 512, "register split must equal the launch budget");

__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

template <int D, int MASK>
__global__ void __launch_bounds__(kBwdThreads, 1)
    fa_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                  const __grid_constant__ CUtensorMap tm_dq, const __grid_constant__ CUtensorMap tm_lse2,
                  const __grid_constant__ CUtensorMap tm_dsum, const BwdParams p) {
  using L = BwdLayout<D>;
  constexpr int QS = L::kStages;
  constexpr int KCH = D / 64;

  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_u32(smem) & 1023u) != 0u) {  // uniform over the CTA: nothing started yet
    if (threadIdx.x == 0) atomicOr(&g_device_error, FA_DEVERR_SMEM_ALIGN);
    return;
  }

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* kv_full = bars;
  uint64_t* qd_full = kv_full + 1;      // [QS]
  uint64_t* qd_empty = qd_full + QS;    // [QS]
  uint64_t* s_full = qd_empty + QS;     // [2]
  uint64_t* dp_full = s_full + 2;       // [2]
  uint64_t* p_full = dp_full + 2;       // [2]
  uint64_t* ds_full = p_full + 2;       // [2]
  uint64_t* dq_full = ds_full + 2;      // [2]
  uint64_t* dq_empty = dq_full + 2;     // [2]
  uint64_t* y_done = dq_empty + 2;      // [2] dK of the buffer's last iteration done
  uint64_t* acc_full = y_done + 2;
  uint64_t* mma_done = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

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
  const int n_q = (N + 63) / 64;
  // 64-query tiles [i_start, i_end) that see a key of this tile; never empty,
  // since key 128*j < N sees itself.
  int i_start = 0, i_end = n_q;
  if (MASK == kMaskCausal) i_start = 2 * j;
  if (MASK == kMaskBand) {
    i_start = max(0, j * 128 - p.wr) / 64;
    i_end = min(n_q, min(j * 128 + 127 + p.wl, N - 1) / 64 + 1);
  }
  const int n_iq = i_end - i_start;  // query tiles per head
  const int n_it = group * n_iq;
  auto q_start = [&](int it) { return (i_start + it % n_iq) * 64; };
  auto q_head = [&](int it) { return qh0 + it / n_iq; };

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < QS; ++s) {
      mbar_init(qd_full + s, 1);
      mbar_init(qd_empty + s, 2);  // one release per MMA issuer
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full + b, 1);
      mbar_init(dp_full + b, 1);
      mbar_init(p_full + b, 4);   // one arrival per warp of the elementwise group
      mbar_init(ds_full + b, 4);
      mbar_init(dq_full + b, 1);
      mbar_init(dq_empty + b, 4);
      mbar_init(y_done + b, 1);
    }
    mbar_init(acc_full, 2);   // last dV (X) and last dK (Y)
    mbar_init(mma_done, 3);   // one per MMA issuer
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int wg = warp >> 2;
  // TMEM columns: S[b] at 64*b, dP[b] at 128 + 64*b, dV at 256, dK at 256 + D.
  const uint32_t t_dv = 256, t_dk = 256 + D;
  constexpr uint32_t kStageTx = 2 * L::kQT + 512;

  if (wg == 0) setmaxnreg_dec<kRegCtl>();
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      prefetch_tmap(&tm_do);
      prefetch_tmap(&tm_dq);
      prefetch_tmap(&tm_lse2);
      prefetch_tmap(&tm_dsum);
      mbar_arrive_expect_tx(kv_full, 2 * L::kKV);
      for (int c = 0; c < KCH; ++c) {
        tma_load_3d(smem + L::kK + c * 16384, &tm_k, kv_full, c * 64, s0 + j * 128, kvh);
        tma_load_3d(smem + L::kV + c * 16384, &tm_v, kv_full, c * 64, s0 + j * 128, kvh);
      }
      int issued = 0;
      for (int it = 0; it < n_it; ++it) {
        const int s = it % QS, u = it / QS;
        if (it >= QS && !wait_parity(qd_empty + s, (u - 1) & 1, abort_flag)) break;
        const int q0 = q_start(it), bhq = q_head(it);
        uint8_t* st = smem + L::kStat + s * 512;
        mbar_arrive_expect_tx(qd_full + s, kStageTx);
        for (int c = 0; c < KCH; ++c) {
          tma_load_3d(smem + L::kQ + s * L::kQT + c * 8192, &tm_q, qd_full + s, c * 64, s0 + q0, bhq);
          tma_load_3d(smem + L::kDO + s * L::kQT + c * 8192, &tm_do, qd_full + s, c * 64, s0 + q0, bhq);
        }
        tma_load_2d(st, &tm_lse2, qd_full + s, stat0 + q0, bhq);
        tma_load_2d(st + 256, &tm_dsum, qd_full + s, stat0 + q0, bhq);
        issued = it + 1;
      }
      wait_parity_drain(kv_full, 0);
      for (int it = max(0, issued - QS); it < issued; ++it) wait_parity_drain(qd_full + it % QS, (it / QS) & 1);
    }
  } else if (warp >= 1 && warp <= 3) {
    // ------------------------------------------------------- MMA issuers
    // Issuing one tcgen05.mma costs the issuing thread about 100 cycles
    // (measured), longer than a 128 x 64 x 16 product takes on the tensor
    // core, so three threads share the 32 instructions of an iteration:
    // X (warp 1) issues S^T and dV, Y (warp 2) dP^T and dK, Z (warp 3) dQ^T.
    // X and Y meet at TMEM buffer S[b]: S^T(it+2) may overwrite it only after
    // dK(it) has read dS^T from it (barrier y_done[b]; dV(it) is X's own and
    // runs first). X and Y read the Q/dO stage, so qd_empty takes one release
    // from each.
    if (lane == 0) {
      const bool is_x = (warp == 1), is_z = (warp == 3);
      constexpr uint32_t kIdST = idesc_bf16(128, 64, 0, 0);  // S^T, dP^T: K-major A and B
      constexpr uint32_t kIdAcc = idesc_bf16(128, D, 0, 1);  // dV, dK: A TMEM, B MN-major
      constexpr uint32_t kIdDQ = idesc_bf16(D, 64, 1, 1);    // dQ^T: A, B MN-major
      const uint32_t k_addr = smem_u32(smem + L::kK);
      const uint32_t v_addr = smem_u32(smem + L::kV);
      const uint32_t q_addr = smem_u32(smem + L::kQ);
      const uint32_t do_addr = smem_u32(smem + L::kDO);
      const uint32_t ds_addr = smem_u32(smem + L::kDS);

      // X^T = A_j Y^T, A_j a 128-row K/V tile, Y a 64-row Q/dO tile (both K-major).
      auto issue_t = [&](uint32_t d_col, uint32_t a_base, uint32_t b_base) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t oa = (kk >> 2) * 16384 + (kk & 3) * 32;
          const uint32_t ob = (kk >> 2) * 8192 + (kk & 3) * 32;
          mma_ss(tmem + d_col, sdesc_sw128(a_base + oa, 16, 1024), sdesc_sw128(b_base + ob, 16, 1024), kIdST,
                 kk > 0);
        }
      };
      // acc += X^T(TMEM, 64 query columns as bf16) * Y (Y a 64-row tile, MN-major)
      auto issue_acc = [&](uint32_t d_col, uint32_t a_col, uint32_t b_base, bool acc) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ts(tmem + d_col, tmem + a_col + kk * 8, sdesc_sw128(b_base + kk * 2048, 8192, 1024), kIdAcc,
                 (acc || kk > 0) ? 1u : 0u);
      };
      auto issue_dq = [&](int b) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tmem + 128 + 64 * b, sdesc_sw128(k_addr + kk * 2048, 16384, 1024),
                 sdesc_sw128(ds_addr + b * L::kDSTile + kk * 2048, 8192, 1024), kIdDQ, kk > 0);
      };

      bool ok = wait_parity(kv_full, 0, abort_flag) && (is_z || wait_parity(qd_full, 0, abort_flag));
      if (ok && !is_z) {
        tc_fence_after();
        if (is_x) {
          issue_t(0, k_addr, q_addr);
          mma_commit(s_full + 0);
        } else {
          issue_t(128, v_addr, do_addr);
          mma_commit(dp_full + 0);
        }
      }
      for (int it = 0; ok && it < n_it; ++it) {
        const int b = it & 1, s = it % QS;
        const int nb = b ^ 1, ns = (it + 1) % QS;
        const bool has_next = it + 1 < n_it;
        if (is_z) {
          if (!(ok = wait_parity(ds_full + b, (it >> 1) & 1, abort_flag))) break;
          tc_fence_after();
          issue_dq(b);
          mma_commit(dq_full + b);
        } else if (is_x) {
          if (has_next) {
            if (!(ok = wait_parity(qd_full + ns, ((it + 1) / QS) & 1, abort_flag))) break;
            if (it >= 1 && !(ok = wait_parity(y_done + nb, ((it - 1) >> 1) & 1, abort_flag))) break;
            tc_fence_after();
            issue_t(64 * nb, k_addr, q_addr + ns * L::kQT);
            mma_commit(s_full + nb);
          }
          if (!(ok = wait_parity(p_full + b, (it >> 1) & 1, abort_flag))) break;
          tc_fence_after();
          issue_acc(t_dv, 64 * b, do_addr + s * L::kQT, it > 0);
          mma_commit(qd_empty + s);
        } else {
          if (has_next) {
            if (!(ok = wait_parity(qd_full + ns, ((it + 1) / QS) & 1, abort_flag))) break;
            if (it >= 1 && !(ok = wait_parity(dq_empty + nb, ((it - 1) >> 1) & 1, abort_flag))) break;
            tc_fence_after();
            issue_t(128 + 64 * nb, v_addr, do_addr + ns * L::kQT);
            mma_commit(dp_full + nb);
          }
          if (!(ok = wait_parity(ds_full + b, (it >> 1) & 1, abort_flag))) break;
          tc_fence_after();
          issue_acc(t_dk, 64 * b + 32, q_addr + s * L::kQT, it > 0);
          mma_commit(y_done + b);
          mma_commit(qd_empty + s);
        }
      }
      if (ok && !is_z) mma_commit(acc_full);
      // Let every MMA the issuers started finish before TMEM is freed.
      mma_commit(mma_done);
      wait_parity_drain(mma_done, 0);
    }
  } else if (wg >= 2) {
    // ---------------------------------------- elementwise (thread = key row)
    // Group e handles iterations it = e, e+2, ... with TMEM/smem buffer b = e.
    setmaxnreg_inc<kRegElem>();
    const int e = wg - 2;
    const int quarter = warp & 3;
    const int k = quarter * 32 + lane;
    const int kj = j * 128 + k;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const float lam = p.scale_log2;
    const float scale = p.scale;
    const int b = e;
    const uint32_t tS = tmem + lane_off + 64 * b;
    const uint32_t tP = tmem + lane_off + 128 + 64 * b;
    uint8_t* ds_row = smem + L::kDS + b * L::kDSTile + k * 128;
    bool ok = true;
    for (int it = e; it < n_it; it += 2) {
      const int s = it % QS;
      const int q0 = q_start(it);
      ok = __all_sync(0xffffffffu, wait_parity(qd_full + s, (it / QS) & 1, abort_flag) &&
                                       wait_parity(s_full + b, (it >> 1) & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      const float4* lse2 = reinterpret_cast<const float4*>(smem + L::kStat + s * 512);
      const float4* dd = lse2 + 16;
      const bool edge = (q0 + 64 > N) || (j * 128 + 128 > N) || (MASK == kMaskCausal && j * 128 + 127 > q0) ||
                        (MASK == kMaskBand && (j * 128 + 127 > q0 + p.wr || j * 128 < q0 + 63 - p.wl));
      float pr[64];
      {
        uint32_t sv[64];
        tmem_ld32(tS, sv);
        tmem_ld32(tS + 32, sv + 32);
        tmem_wait_ld();
#pragma unroll
        for (int c4 = 0; c4 < 16; ++c4) {
          const float4 l4 = lse2[c4];
          pr[4 * c4 + 0] = ex2(fmaf(__uint_as_float(sv[4 * c4 + 0]), lam, -l4.x));
          pr[4 * c4 + 1] = ex2(fmaf(__uint_as_float(sv[4 * c4 + 1]), lam, -l4.y));
          pr[4 * c4 + 2] = ex2(fmaf(__uint_as_float(sv[4 * c4 + 2]), lam, -l4.z));
          pr[4 * c4 + 3] = ex2(fmaf(__uint_as_float(sv[4 * c4 + 3]), lam, -l4.w));
        }
      }
      if (edge) {
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const int qi = q0 + c;
          const bool vis = (qi < N) && (kj < N) && (MASK != kMaskCausal || kj <= qi) &&
                           (MASK != kMaskBand || (kj >= qi - p.wl && kj <= qi + p.wr));
          if (!vis) pr[c] = 0.f;
        }
      }
      {
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) pk[c] = pack_bf16(pr[2 * c], pr[2 * c + 1]);
        tmem_st32(tS, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full + b);

      // dS tile b was last read by dQ^T(it - 2), which finished before the
      // drain released its TMEM buffer and so before dP^T(it) was issued.
      ok = __all_sync(0xffffffffu, wait_parity(dp_full + b, (it >> 1) & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t dp[32];
        tmem_ld32(tP + 32 * h, dp);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4) {
          const float4 d4 = dd[8 * h + c4];
          const int q = 32 * h + 4 * c4;
          const float s0 = pr[q + 0] * (__uint_as_float(dp[4 * c4 + 0]) - d4.x) * scale;
          const float s1 = pr[q + 1] * (__uint_as_float(dp[4 * c4 + 1]) - d4.y) * scale;
          const float s2 = pr[q + 2] * (__uint_as_float(dp[4 * c4 + 2]) - d4.z) * scale;
          const float s3 = pr[q + 3] * (__uint_as_float(dp[4 * c4 + 3]) - d4.w) * scale;
          pk[2 * c4] = pack_bf16(s0, s1);
          pk[2 * c4 + 1] = pack_bf16(s2, s3);
        }
        tmem_st16(tS + 32 + 16 * h, pk);
        // Row k of the [128 keys][64 queries] dS tile, 128-byte swizzle:
        // 16-byte chunk c (queries 8c..8c+7) lives at chunk c ^ (k & 7).
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
      if (lane == 0) mbar_arrive(ds_full + b);
    }
    // -------------------------------------- epilogue: group 0 dV, group 1 dK
    if (ok) {
      ok = __all_sync(0xffffffffu, wait_parity(acc_full, 0, abort_flag));
      if (ok) {
        tc_fence_after();
        const bool valid = kj < N;
        const int kv = valid ? kj : 0;
        // dK/dV row of key kj, in units of D elements.
        const size_t row = packed ? static_cast<size_t>(s0 + kv) * p.Hkv + kvh : static_cast<size_t>(bkv) * N + kv;
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(e ? p.dk : p.dv) + row * D;
        float* acc = (e ? p.dk_acc : p.dv_acc) + row * D;
        const uint32_t col = e ? t_dk : t_dv;
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_off + col + c, v);
          tmem_wait_ld();
          if (valid && p.n_split > 1) {
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
  } else if (wg == 1) {
    // ------------------------------------------------- dQ drain (warps 4-7)
    // dQ_i^T sits in TMEM with the head-dim index on lanes and the 64 queries
    // on columns. The drain copies each half (32 queries) into its own fp32
    // [32][D] staging buffer and one TMA reduce-add per half adds it into the
    // fp32 accumulator; the TMA engine streams the reduction to L2 while the
    // warps stage the next half, waiting only for that buffer's previous read.
    setmaxnreg_dec<kRegDrain>();
    const int quarter = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    // M = D = 128 uses every lane; M = 64 uses lanes 0-15 of each quarter.
    const int drow = (D == 128) ? quarter * 32 + lane : quarter * 16 + lane;
    const bool holds = (D == 128) || (lane < 16);
    const bool leader = (warp == 4 && lane == 0);
    bool ok = true;
    // Every drain warp runs all 4*n_it named barriers, even after an abort
    // (work is skipped instead), so no warp can be left waiting at one.
    for (int it = 0; it < n_it; ++it) {
      const int b = it & 1;
      if (ok) ok = __all_sync(0xffffffffu, wait_parity(dq_full + b, (it >> 1) & 1, abort_flag));
      uint32_t v[64];
      if (ok) {
        tc_fence_after();
        tmem_ld32(tmem + lane_off + 128 + 64 * b, v);
        tmem_ld32(tmem + lane_off + 128 + 64 * b + 32, v + 32);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(dq_empty + b);
      }
      const int q0 = q_start(it), bhq = q_head(it);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float* stg = reinterpret_cast<float*>(smem + L::kStg + h * L::kStgHalf);
        // Groups go out in order (it-1, 0), (it-1, 1), (it, 0), ...: at most one
        // pending means the previous read of this half's buffer is done.
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
