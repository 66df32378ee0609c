// fa_fwd.cuh - fused attention forward for sm_100a (TMA + tcgen05 + TMEM).
//
// Method: "FlashAttention原理：从原始Attention到FlashAttention"
// (blog.csdn.net/qq_43527718), sections 二.5-二.7, and "FlashAttention：优化大模型
// 训练的内存与计算效率" (cnnetsun.cn), sections 2.1-2.2. Q is tiled against K/V
// blocks held on chip; each block's scores are merged into the output with a
// running row maximum m and running row sum l; O is divided by l once at the
// end (the second FlashAttention's cut of non-matmul work, blog section 二.7);
// query tiles form the outer loop and key/value tiles the inner loop (same
// section); tiles wholly above the causal diagonal are never visited (same
// section, third point). Only O and lse reach global memory. A local window
// (the band i - wl <= j <= i + wr, "Local-Window" in cnnetsun.cn section 6.1)
// visits only the K/V tiles the band touches, each query tile its own range.
//
// Layouts. Fixed length: Q, O [B, H, N, D], K, V [B, Hkv, N, D]; the tensor
// maps index (column, row, batch*head). Packed variable length: Q, O
// [T, H, D], K, V [T, Hkv, D] with sequence b in rows [cu[b], cu[b+1]); the
// maps index (column, packed row, head), and a CTA adds its sequence's first
// row to every row coordinate. lse is [B, H, N] or [H, T].
//
// One CTA owns two 128-row query tiles of one (batch, head) and streams the
// K/V tiles of that head through a shared-memory ring:
//   warp 0      TMA producer: Q0, K_0, Q1 (each query tile under its own
//               barrier, so the first S waits for one tile), then K_j, V_j
//               into a K/V ring.
//   warps 1, 10 MMA issuers (one thread each, taking alternate K/V steps):
//               S_t = Q_t K_j^T into TMEM, then O_t += P_t V_j with P_t read
//               from TMEM. The two tiles alternate so that the tensor core
//               works on one tile while the other tile's softmax runs.
//   warps 2-5   softmax warpgroup of tile 0 (one thread per query row).
//   warps 6-9   softmax warpgroup of tile 1.
// TMEM columns (512 allocated): S0/P0 [0,128), S1/P1 [128,256),
// O0 [256, 256+D), O1 [256+D, 256+2D).
//
// Softmax per row, in log2 units (lambda = scale*log2(e)):
//   m_blk = lambda * max_j S_ij;  if m_blk > m + 8 the running max moves to
//   m_blk and O, l are multiplied by alpha = 2^(m_old - m_new) (else m stays:
//   the result is the same because O and l share the same stale m, and the
//   largest p is at most 2^8);  p_ij = 2^(lambda*S_ij - m);  l = alpha*l + sum p.
//   Epilogue: O /= l;  lse = ln2 * (m + log2 l).
//
// FP8 (FP8 = true, D = 128): Q, K, V are e4m3 codes with per-tensor
// dequantisation scales. S and PV run as kind::f8f6f4 MMAs (K = 32 per
// instruction); the Q and K scales fold into lambda and the V scale into the
// epilogue (o_scale). P is rounded to e4m3 for the PV product (p <= 2^8 < 448,
// the largest e4m3 value); l sums the unrounded p.
#pragma once
#include <cuda.h>

#include <type_traits>

#include "fa_ptx.cuh"

namespace fa {

struct FwdParams {
  void* o;
  float* lse;
  int BH;   // batch * query heads
  int H;    // query heads
  int Hkv;  // K/V heads (H % Hkv == 0; query head h reads K/V head h / (H / Hkv))
  int N;
  int n_pairs;       // ceil(N / 256): CTAs per (batch, head)
  float scale_log2;  // scale * log2(e) (FP8: times the Q and K dequantisation scales)
  float o_scale;     // multiplies O in the epilogue: 1, or the V dequantisation scale (FP8)
  int wl, wr;        // band mask only: key j visible to query i iff i - wl <= j <= i + wr (0 <= wl, wr <= N)
  int sched_groups;  // causal launch order: number of head groups (1 <= sched_groups <= BH)
  const int* cu_seqlens;  // packed variable length: [B + 1] prefix sums of the lengths; else nullptr
  int T;                  // packed rows (variable length only); N is then the longest length
};

template <int D, int ESZ = 2>  // ESZ: bytes per element (2 bf16, 1 e4m3)
struct FwdLayout {
  static constexpr int kRowBytes = D * ESZ;
  static constexpr int kTile = 128 * kRowBytes;               // one 128-row tile
  static constexpr int kChunks = kRowBytes / 128;             // 128-byte column chunks per row
  static constexpr int kKStages = (kRowBytes == 256) ? 2 : 4;  // K ring depth
  static constexpr int kVStages = kKStages;                     // V ring depth
  static constexpr int kQ0 = 0;
  static constexpr int kQ1 = kTile;
  static constexpr int kK = 2 * kTile;
  static constexpr int kV = kK + kKStages * kTile;
  static constexpr int kBar = kV + kVStages * kTile;
  static constexpr int kBytes = kBar + 256;
  static constexpr int kAlloc = kBytes + 1024;  // slack for 1 KB alignment
  static_assert(kAlloc <= 227 * 1024, "shared memory budget");
};

// MMA issuing threads: 1, or 2 taking alternate K/V steps (an eleventh
// warp), so one thread's barrier waits overlap the other's MMA issue.
#ifndef FA_FWD_ISSUERS
#define FA_FWD_ISSUERS 2
#endif
constexpr int kFwdIssuers = FA_FWD_ISSUERS;
constexpr int kFwdThreads = kFwdIssuers == 2 ? 352 : 320;
constexpr int kFwdIssuer2Warp = 10;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// Every kPolyEvery-th column pair of an unmasked tile takes its exponentials
// on the FMA pipe (exp2_fma2) instead of the special-function unit; 0: none.
#ifndef FA_FWD_POLY_EVERY
#define FA_FWD_POLY_EVERY 6
#endif
constexpr int kPolyEvery = FA_FWD_POLY_EVERY;
// P goes to the PV MMA in two halves (1) or at once (0).
#ifndef FA_FWD_SPLIT_P
#define FA_FWD_SPLIT_P 1
#endif
constexpr bool kSplitP = FA_FWD_SPLIT_P != 0;
// The FP8 softmax's share on the FMA pipe: every kPolyEvery8-th group of four
// columns of an unmasked tile (0: none).
#ifndef FA_FWD_FP8_POLY_EVERY
#define FA_FWD_FP8_POLY_EVERY 4
#endif
constexpr int kPolyEvery8 = FA_FWD_FP8_POLY_EVERY;
// Q_0 and Q_1 under one barrier each, Q_1 loaded after K_0, so the first S
// waits for one query tile instead of two (1), or both under one barrier (0).
#ifndef FA_FWD_Q_SPLIT
#define FA_FWD_Q_SPLIT 1
#endif
constexpr bool kQSplit = FA_FWD_Q_SPLIT != 0;
// The epilogue's TMA stores waited for until their shared-memory source has
// been read (1) or until the writes are complete (0).
#ifndef FA_FWD_STORE_WAIT_READ
#define FA_FWD_STORE_WAIT_READ 1
#endif
// TMEM columns of P the softmax packs and stores at a time: 32, 16 or 8.
// Fewer keep fewer packed values live beside the 128 scores.
#ifndef FA_FWD_P_ST_COLS
#define FA_FWD_P_ST_COLS 16
#endif
// The warp index read through a shuffle from lane 0 (1), which marks it, and
// everything derived from it, as the same for all lanes of a warp: the
// compiler can then keep those values in uniform registers instead of the
// per-thread ones the 128 scores need.
#ifndef FA_FWD_UNIFORM_WARP
#define FA_FWD_UNIFORM_WARP 1
#endif
// The thread that initialises the barriers also issues the first Q and K
// loads, before the block-wide barrier (1), or the producer issues them after
// it (0).
#ifndef FA_FWD_EARLY_LOAD
#define FA_FWD_EARLY_LOAD 1
#endif
constexpr bool kEarlyLoad = FA_FWD_EARLY_LOAD != 0;
// The commit that releases V_j's ring stage comes after S_1(j+1) is issued
// (1), so S_1(j+1) is not queued behind it, or between PV_1(j) and S_1(j+1)
// (0).
#ifndef FA_FWD_V_RELEASE_LATE
#define FA_FWD_V_RELEASE_LATE 1
#endif
// With two issuers: the arrive that lets the other issuer start the next step
// comes after S_1(j+1) is issued and committed (1), or just before (0).
#ifndef FA_FWD_TURN_LATE
#define FA_FWD_TURN_LATE 1
#endif

constexpr int kPStCols = FA_FWD_P_ST_COLS;
static_assert(kPStCols == 32 || kPStCols == 16 || kPStCols == 8, "P store width");

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t* r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}
// max(a, b, c) in one instruction.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 2^x for a pair of fp32 values on the FMA pipe, x <= 2^22 (here x <= 8).
// Cody and Waite's range reduction: n = round(x) by adding and subtracting
// 1.5 * 2^23, f = x - n in [-1/2, 1/2], 2^x = 2^n * p(f) with p the degree-3
// polynomial of least maximum relative error on [-1/2, 1/2] (Remez exchange;
// coefficients from csrc/exp2_poly.py, relative error below 7.5e-5 in fp32),
// and 2^n added into p's exponent field. x is clamped below at -125 so the
// result stays a normal number (2^-125 instead of a smaller value or 0).
__device__ __forceinline__ float2 exp2_fma2(float2 x) {
  constexpr float kShift = 12582912.0f;  // 1.5 * 2^23
  constexpr float c0 = 0.99992806f, c1 = 0.69326097f, c2 = 0.24261113f, c3 = 0.05517167f;
  x = make_float2(fmaxf(x.x, -125.f), fmaxf(x.y, -125.f));
  const float2 t = fadd2(x, make_float2(kShift, kShift));
  const float2 f = fsub2(x, fsub2(t, make_float2(kShift, kShift)));
  float2 p = ffma2(make_float2(c3, c3), f, make_float2(c2, c2));
  p = ffma2(p, f, make_float2(c1, c1));
  p = ffma2(p, f, make_float2(c0, c0));
  // The low mantissa bits of t hold n (two's complement); shifted by 23 they
  // land in the exponent field, and the shifter's own bits shift out.
  return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                     __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

template <int D, int MASK, bool OF32, bool FP8 = false>
__global__ void __launch_bounds__(kFwdThreads, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                  const FwdParams p) {
  static_assert(!FP8 || D == 128, "the FP8 forward is built for D = 128");
  constexpr int ESZ = FP8 ? 1 : 2;
  using L = FwdLayout<D, ESZ>;
  constexpr int CW = 128 / ESZ;  // elements per 128-byte chunk
  constexpr int KS = L::kKStages, VS = L::kVStages;
  constexpr int KCH = L::kChunks;  // 128-byte column chunks per row

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  static_assert(8 * (2 + 2 * KS + 2 * VS + 8 + kFwdIssuers + 2) + 8 <= L::kBytes - L::kBar, "barrier area");
  uint64_t* q_full = bars + 0;  // [2]: Q_0, Q_1 (only [0] without kQSplit)
  uint64_t* k_full = bars + 2;
  uint64_t* k_empty = k_full + KS;
  uint64_t* v_full = k_empty + KS;
  uint64_t* v_empty = v_full + VS;
  uint64_t* s_full = v_empty + VS;  // [2]
  uint64_t* p_half = s_full + 2;   // [2] P of keys 0-63 in TMEM (and O rescaled)
  uint64_t* p_full = p_half + 2;   // [2] P of keys 64-127 in TMEM
  uint64_t* o_full = p_full + 2;   // [2] the tile's last PV done (once per CTA)
  uint64_t* mma_done = o_full + 2;  // [kFwdIssuers]
  // [2] with two issuers: turn[i] is arrived on by the other issuer once it
  // has passed every wait of its step, which makes issuer i's next parity
  // waits unambiguous (the phase before each is then known to be complete).
  uint64_t* turn = mma_done + kFwdIssuers;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(turn + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = FA_FWD_UNIFORM_WARP ? __shfl_sync(0xffffffffu, static_cast<int>(threadIdx.x >> 5), 0)
                                      : static_cast<int>(threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;

  // Causal: heads in sched_groups groups, each small enough that its K/V
  // stays in L2 and large enough that its heaviest query tiles (started
  // first) finish with the rest; see grouped_order. Otherwise head-major, so
  // CTAs that read the same K/V run together.
  int pair, bh;
  if (MASK == kMaskCausal) {
    int t;
    grouped_order(static_cast<int>(blockIdx.x), p.BH, p.sched_groups, p.n_pairs, t, bh);
    pair = p.n_pairs - 1 - t;
  } else {
    bh = static_cast<int>(blockIdx.x) / p.n_pairs;
    pair = static_cast<int>(blockIdx.x) % p.n_pairs;
  }
  // This CTA's sequence: its length N and first row s0 in the maps' row
  // dimension, and the Q/O head coordinate hq of the maps.
  const bool packed = p.cu_seqlens != nullptr;
  int N = p.N, s0 = 0;
  const int hq = packed ? bh % p.H : bh;
  if (packed) seq_range(p.cu_seqlens, bh / p.H, p.T, p.N, s0, N);
  const int q0 = pair * 256;
  if (q0 >= N) return;  // past the end of a shorter sequence: the whole CTA leaves
  const int n_kv = (N + 127) / 128;
  // K/V tiles [lo, hi) that query tile t needs. The CTA streams tiles j0 + j,
  // j in [0, J); tile t takes part in steps [a_t, b_t) of that stream. The
  // two ranges overlap or touch (the diagonal tile of query tile 0 reaches
  // the first tile query tile 1 needs), so the stream has no gaps.
  int a_t[2], b_t[2], j0 = 0;
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int qs = q0 + 128 * t;
    int lo = 0, hi = 0;
    if (qs < N) {
      hi = n_kv;
      if (MASK == kMaskCausal) hi = min(n_kv, qs / 128 + 1);
      if (MASK == kMaskBand) {
        lo = max(0, qs - p.wl) / 128;
        hi = min(n_kv, (min(qs + 127, N - 1) + p.wr) / 128 + 1);
      }
    }
    if (t == 0) j0 = lo;
    a_t[t] = (hi > lo) ? lo - j0 : 0;
    b_t[t] = (hi > lo) ? hi - j0 : 0;
  }
  const int J = max(b_t[0], b_t[1]);
  // Only the bf16-in, bf16-out instantiations take the early first load: in
  // the fp32-O and FP8 ones the moved code makes the compiler spill registers.
  constexpr bool kEarly = kEarlyLoad && !OF32 && !FP8;

  // K/V head of this query head (grouped-query attention; equal for MHA).
  const int bkv = (packed ? 0 : (bh / p.H) * p.Hkv) + (bh % p.H) / (p.H / p.Hkv);
  auto load_q = [&](int t) {
    uint64_t* bar = q_full + (kQSplit ? t : 0);
    for (int c = 0; c < KCH; ++c)
      tma_load_3d(smem + (t ? L::kQ1 : L::kQ0) + c * 16384, &tm_q, bar, c * CW, s0 + q0 + 128 * t, hq);
  };
  auto start_q = [&]() {  // the barriers' transaction counts, then Q_0 (and Q_1 without kQSplit)
    if (kQSplit) {
      mbar_arrive_expect_tx(q_full + 0, L::kTile);
      mbar_arrive_expect_tx(q_full + 1, L::kTile);
      load_q(0);
    } else {
      mbar_arrive_expect_tx(q_full, 2 * L::kTile);
      load_q(0);
      load_q(1);
    }
  };
  auto load_k = [&](int j) {
    const int sk = j % KS;
    mbar_arrive_expect_tx(k_full + sk, L::kTile);
    for (int c = 0; c < KCH; ++c)
      tma_load_3d(smem + L::kK + sk * L::kTile + c * 16384, &tm_k, k_full + sk, c * CW, s0 + (j0 + j) * 128, bkv);
  };

  if (threadIdx.x == 0) {
    mbar_init(q_full + 0, 1);
    mbar_init(q_full + 1, 1);
    for (int s = 0; s < KS; ++s) {
      mbar_init(k_full + s, 1);
      mbar_init(k_empty + s, 1);
    }
    for (int s = 0; s < VS; ++s) {
      mbar_init(v_full + s, 1);
      mbar_init(v_empty + s, 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(s_full + t, 1);
      mbar_init(p_half + t, 128);
      mbar_init(p_full + t, 128);
      mbar_init(o_full + t, 1);
    }
    for (int i = 0; i < kFwdIssuers; ++i) mbar_init(mma_done + i, 1);
    mbar_init(turn + 0, 1);
    mbar_init(turn + 1, 1);
    *abort_flag = 0;
    fence_barrier_init();
    if (kEarly) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      start_q();
      load_k(0);
    }
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      if (!kEarly) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        start_q();
      }
      int k_issued = 0, v_issued = 0;
      for (int j = 0; j < J; ++j) {
        const int sk = j % KS, sv = j % VS;
        if (j >= KS && !wait_parity(k_empty + sk, (j / KS - 1) & 1, abort_flag)) break;
        if (!(kEarly && j == 0)) load_k(j);  // else issued with the barriers' setup
        k_issued = j + 1;
        if (kQSplit && j == 0) load_q(1);
        if (j >= VS && !wait_parity(v_empty + sv, (j / VS - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(v_full + sv, L::kTile);
        for (int c = 0; c < KCH; ++c)
          tma_load_3d(smem + L::kV + sv * L::kTile + c * 16384, &tm_v, v_full + sv, c * CW, s0 + (j0 + j) * 128, bkv);
        v_issued = j + 1;
      }
      // Every copy this thread started must land before the CTA exits.
      wait_parity_drain(q_full + 0, 0);
      if (kQSplit) wait_parity_drain(q_full + 1, 0);
      for (int j = max(0, k_issued - KS); j < k_issued; ++j) wait_parity_drain(k_full + j % KS, (j / KS) & 1);
      for (int j = max(0, v_issued - VS); j < v_issued; ++j) wait_parity_drain(v_full + j % VS, (j / VS) & 1);
    }
  } else if (warp == 1 || (kFwdIssuers == 2 && warp == kFwdIssuer2Warp)) {
    // ---------------------------------------------------------- MMA issuer
    // Issuer `me` takes K/V steps j = me, me + kFwdIssuers, ...: PV_t(j) of
    // both tiles, then S_t(j+1). Each tile's PV_t(j) and S_t(j+1) come from
    // one thread, so S_t(j+1) overwrites P_t(j) only after PV_t(j) read it;
    // everything that crosses issuers goes through a barrier whose commit
    // covers all earlier MMAs of the committing thread (s_full_t(j+1) covers
    // PV_t(j), so PV_t(j+1) and the O rescale before it follow PV_t(j)).
    // Between a P hand-over and the S that follows it the thread issues only
    // MMAs: the commit that frees V_j's stage and the other issuer's go-ahead
    // come after S_1(j+1), off each tile's chain P -> PV -> S -> softmax.
    const int me = warp == 1 ? 0 : 1;
    if (lane == 0) {
      // S: Q, K both K-major. PV: P from TMEM, V MN-major.
      constexpr uint32_t kIdS = FP8 ? idesc_e4m3(128, 128, 0, 0) : idesc_bf16(128, 128, 0, 0);
      constexpr uint32_t kIdO = FP8 ? idesc_e4m3(128, D, 0, 1) : idesc_bf16(128, D, 0, 1);
      const uint32_t q_addr[2] = {smem_u32(smem + L::kQ0), smem_u32(smem + L::kQ1)};
      const uint32_t k_addr = smem_u32(smem + L::kK);
      const uint32_t v_addr = smem_u32(smem + L::kV);

      auto issue_s = [&](int t, int stage) {
        const uint32_t ka = k_addr + stage * L::kTile;
        // Each MMA consumes 32 bytes of every row (16 bf16 or 32 e4m3).
#pragma unroll
        for (int kk = 0; kk < L::kRowBytes / 32; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          const uint64_t da = sdesc_sw128(q_addr[t] + off, 16, 1024), db = sdesc_sw128(ka + off, 16, 1024);
          if (FP8)
            mma_ss_f8(tmem + t * 128, da, db, kIdS, kk > 0);
          else
            mma_ss(tmem + t * 128, da, db, kIdS, kk > 0);
        }
      };
      // PV over keys [64 half, 64 half + 64): the softmax hands P over in two
      // halves, so the product over the first half overlaps the exponentials
      // of the second.
      auto issue_pv = [&](int t, int stage, bool acc, int half) {
        const uint32_t va = v_addr + stage * L::kTile;
        // Each MMA takes 32 bytes of P per row (8 TMEM columns: 16 bf16 or 32
        // e4m3 keys) and the matching 16 or 32 rows of V.
#pragma unroll
        for (int kk = half * 2 * ESZ; kk < (half + 1) * 2 * ESZ; ++kk) {
          const uint64_t dv = sdesc_sw128(va + kk * (32 / ESZ) * 128, 16384, 1024);
          if (FP8)
            mma_ts_f8(tmem + 256 + t * D, tmem + t * 128 + kk * 8, dv, kIdO, (acc || kk > 0) ? 1u : 0u);
          else
            mma_ts(tmem + 256 + t * D, tmem + t * 128 + kk * 8, dv, kIdO, (acc || kk > 0) ? 1u : 0u);
        }
      };

      bool ok = me == 0 ? (wait_parity(q_full, 0, abort_flag) && wait_parity(k_full, 0, abort_flag)) : true;
      if (ok && me == 0) {
        tc_fence_after();
#pragma unroll
        for (int t = 0; t < 2; ++t)
          if (a_t[t] == 0 && b_t[t] > 0) {
            if (kQSplit && t == 1) {
              if (!(ok = wait_parity(q_full + 1, 0, abort_flag))) break;
              tc_fence_after();
            }
            issue_s(t, 0);
            mma_commit(s_full + t);
          }
        if (ok) mma_commit(k_empty + 0);
      }
      for (int j = me; ok && j < J; j += kFwdIssuers) {
        if (kFwdIssuers == 2 && j > 0) {
          // Issuer 0's k-th step follows issuer 1's (k-1)-th, issuer 1's
          // k-th follows issuer 0's k-th.
          const int k = j >> 1;
          if (!(ok = wait_parity(turn + me, (me == 0 ? k - 1 : k) & 1, abort_flag))) break;
        }
        const int s = j % VS;
        if (!(ok = wait_parity(v_full + s, (j / VS) & 1, abort_flag))) break;
        tc_fence_after();
        const int jn = j + 1, sn = jn % KS;
        bool k_next = false;
        // Unrolled, so the per-tile ranges and addresses stay in registers.
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (j >= a_t[t] && j < b_t[t]) {
            if (!(ok = wait_parity(p_half + t, (j - a_t[t]) & 1, abort_flag))) break;
            tc_fence_after();
            issue_pv(t, s, j > a_t[t], 0);
            if (!(ok = wait_parity(p_full + t, (j - a_t[t]) & 1, abort_flag))) break;
            tc_fence_after();
            issue_pv(t, s, true, 1);
            // The epilogue's signal; within the loop the softmax relies on
            // s_full instead (a commit covers every earlier MMA of this
            // thread, so S_t(j+1) done means PV_t(j) done).
            if (j + 1 == b_t[t]) mma_commit(o_full + t);
          }
          if (t == 1 && !FA_FWD_V_RELEASE_LATE) mma_commit(v_empty + s);
          if (jn >= a_t[t] && jn < b_t[t]) {
            if (!k_next) {
              if (!(ok = wait_parity(k_full + sn, (jn / KS) & 1, abort_flag))) break;
              tc_fence_after();
              k_next = true;
            }
            // Query tile 1 joining the stream after the first step (a band).
            if (kQSplit && t == 1 && jn == a_t[1]) {
              if (!(ok = wait_parity(q_full + 1, 0, abort_flag))) break;
              tc_fence_after();
            }
            // Every wait of this step is behind us: the other issuer may
            // start on the next step (after S_1(j+1) is queued, with
            // FA_FWD_TURN_LATE, so that arrive is not on tile 1's chain).
            if (kFwdIssuers == 2 && t == 1 && !FA_FWD_TURN_LATE) mbar_arrive(turn + (1 - me));
            issue_s(t, sn);
            mma_commit(s_full + t);
            if (kFwdIssuers == 2 && t == 1 && FA_FWD_TURN_LATE) mbar_arrive(turn + (1 - me));
          } else if (kFwdIssuers == 2 && t == 1) {
            mbar_arrive(turn + (1 - me));
          }
          if (t == 1 && FA_FWD_V_RELEASE_LATE) mma_commit(v_empty + s);
        }
        if (ok && jn < J) mma_commit(k_empty + sn);
      }
      // Let every MMA this thread issued finish before TMEM is freed.
      mma_commit(mma_done + me);
      wait_parity_drain(mma_done + me, 0);
    }
  } else {
    // ------------------------------------------------------------- softmax
    const int t = (warp - 2) >> 2;
    const int quarter = warp & 3;  // TMEM lane quarter this warp may access
    const int r = quarter * 32 + lane;
    const int qi = q0 + 128 * t + r;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + t * 128;
    const uint32_t tO = tmem + lane_off + 256 + t * D;
    const int a_me = t ? a_t[1] : a_t[0];  // selects, not a local-memory index
    const int nt = (t ? b_t[1] : b_t[0]) - a_me;
    const float lam = p.scale_log2;

    float m = -INFINITY;  // running max, log2 units
    float l = 0.f;        // running sum
    bool ok = true;
    for (int j = 0; j < nt; ++j) {
      ok = __all_sync(0xffffffffu, wait_parity(s_full + t, j & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      float s[128];
      {
        uint32_t sr[128];
        tmem_ld64(tS + 0, sr + 0);
        tmem_ld64(tS + 64, sr + 64);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 128; ++c) s[c] = __uint_as_float(sr[c]);
      }
      const int kb = (j0 + a_me + j) * 128;
      // A tile the mask cuts: this row sees keys kb + [lo_m, hi_m).
      bool masked = false;
      int lo_m = 0, hi_m = 128;
      if (MASK == kMaskBand) {
        const int qs = q0 + 128 * t;
        if (kb + 128 > N || kb + 127 > qs + p.wr || kb < qs + 127 - p.wl) {
          masked = true;
          hi_m = min(N - kb, qi + p.wr - kb + 1);
          lo_m = qi - p.wl - kb;
        }
      } else if (kb + 128 > N || (MASK == kMaskCausal && kb + 127 > q0 + 128 * t)) {
        masked = true;
        hi_m = N - kb;
        if (MASK == kMaskCausal) hi_m = min(hi_m, qi - kb + 1);
      }
      auto mask_cols = [&](auto c0, auto c1) {
#pragma unroll
        for (int c = decltype(c0)::value; c < decltype(c1)::value; ++c)
          if (c >= hi_m || c < lo_m) s[c] = -INFINITY;
      };
      if (masked) mask_cols(std::integral_constant<int, 0>{}, std::integral_constant<int, 128>{});
      // Row max with three-input max instructions, in four chains.
      float mx0 = fmax3(s[0], s[1], s[2]), mx1 = fmax3(s[3], s[4], s[5]), mx2 = s[6], mx3 = s[7];
#pragma unroll
      for (int c = 8; c < 128; c += 8) {
        mx0 = fmax3(mx0, s[c], s[c + 1]);
        mx1 = fmax3(mx1, s[c + 2], s[c + 3]);
        mx2 = fmax3(mx2, s[c + 4], s[c + 5]);
        mx3 = fmax3(mx3, s[c + 6], s[c + 7]);
      }
      const float m_blk = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * lam;
      float alpha = 1.f;
      bool rescale = false;
      if (m_blk > m + kRescaleThreshold) {
        alpha = ex2(m - m_blk);  // 0 on the first visited block (m = -inf)
        m = m_blk;
        rescale = true;
      }
      // O is rescaled before the first half of P is handed over: PV_j
      // accumulates into it from then on. PV_{j-1} is done: S_j's commit,
      // waited for above, covers every MMA the issuer started before it.
      auto rescale_o = [&]() {
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          uint32_t ov[32];
          tmem_ld32(tO + c, ov);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
          tmem_st32(tO + c, ov);
        }
      };
      // A band can hide a whole tile from some rows: while a row has seen no
      // visible key its m is -inf and its p must come out 0, not NaN.
      auto neg_max = [&]() { return (MASK == kMaskBand && m == -INFINITY) ? 0.f : -m; };
      const float2 lam2 = make_float2(lam, lam);
      float2 rs = make_float2(0.f, 0.f);
      if (FP8) {
        if (j > 0 && __any_sync(0xffffffffu, rescale)) rescale_o();
        const float neg_m = neg_max();
        const float2 negm2 = make_float2(neg_m, neg_m);
        // Four e4m3 probabilities per TMEM column: P fills 32 columns. In
        // unmasked tiles every kPolyEvery8-th column's four exponentials run
        // on the FMA pipe; e4m3 rounding of P (2^-4 relative) dwarfs the
        // polynomial's error.
        uint32_t pk[32];
        auto quads = [&](auto use_poly) {
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float2 x0 = ffma2(make_float2(s[4 * c], s[4 * c + 1]), lam2, negm2);
            const float2 x1 = ffma2(make_float2(s[4 * c + 2], s[4 * c + 3]), lam2, negm2);
            float2 p01, p23;
            if (decltype(use_poly)::value && c % kPolyEvery8 == kPolyEvery8 - 1) {
              p01 = exp2_fma2(x0);
              p23 = exp2_fma2(x1);
            } else {
              p01 = make_float2(ex2(x0.x), ex2(x0.y));
              p23 = make_float2(ex2(x1.x), ex2(x1.y));
            }
            rs = fadd2(rs, p01);
            rs = fadd2(rs, p23);
            pk[c] = pack_e4m3x4(p01.x, p01.y, p23.x, p23.y);
          }
        };
        if (kPolyEvery8 > 0 && !masked)
          quads(std::true_type{});
        else
          quads(std::false_type{});
        tmem_st32(tS + 0, pk);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(p_half + t);
        mbar_arrive(p_full + t);
      } else {
        // Tiles without masking send some column pairs through the FMA-pipe
        // exp2 (exp2_fma2), which takes load off the special-function unit;
        // masked tiles keep every exponential on ex2, which gives exactly 0
        // for -inf.
        // Pairs [W q, W q + W) into W packed columns, stored at once.
        auto part = [&](auto use_poly, int q, float neg_m, float2& acc) {
          constexpr int W = kPStCols;
          const float2 negm2 = make_float2(neg_m, neg_m);
          uint32_t pk[W];
#pragma unroll
          for (int cc = 0; cc < W; ++cc) {
            const int c = W * q + cc;
            const float2 x = ffma2(make_float2(s[2 * c], s[2 * c + 1]), lam2, negm2);
            float2 pp;
            if (decltype(use_poly)::value && c % kPolyEvery == kPolyEvery - 1)
              pp = exp2_fma2(x);
            else
              pp = make_float2(ex2(x.x), ex2(x.y));
            acc = fadd2(acc, pp);
            pk[cc] = pack_bf16(pp.x, pp.y);
          }
          if (W == 32)
            tmem_st32(tS + W * q, pk);
          else if (W == 16)
            tmem_st16(tS + W * q, pk);
          else
            tmem_st8(tS + W * q, pk);
        };
        // After each half of P: make the stores visible to the PV MMA, then
        // hand the half over (both halves at once without kSplitP).
        auto handover = [&](int hh) {
          if (hh == 1 || kSplitP) {
            tmem_wait_st();
            tc_fence_before();
            if (hh == 0 || !kSplitP) mbar_arrive(p_half + t);
            if (hh == 1) mbar_arrive(p_full + t);
          }
        };
        auto run = [&](auto use_poly) {
          if (j > 0 && __any_sync(0xffffffffu, rescale)) rescale_o();
          const float neg_m = neg_max();
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
            for (int q = 0; q < 32 / kPStCols; ++q) part(use_poly, hh * (32 / kPStCols) + q, neg_m, rs);
            handover(hh);
          }
        };
        if (kPolyEvery > 0 && !masked)
          run(std::true_type{});
        else
          run(std::false_type{});
      }
      l = l * alpha + (rs.x + rs.y);
    }

    // ------------------------------------------------------------ epilogue
    if (ok && nt > 0) {
      ok = __all_sync(0xffffffffu, wait_parity(o_full + t, 0, abort_flag));
      if (ok) {
        tc_fence_after();
        const float inv_l = (FP8 ? p.o_scale : 1.f) / l;
        const bool valid = qi < N;
        const int qv = valid ? qi : 0;
        // O row (units of D elements) and lse index of query qi.
        const size_t row = packed ? static_cast<size_t>(s0 + qv) * p.H + hq : static_cast<size_t>(bh) * N + qv;
        const size_t li = packed ? static_cast<size_t>(hq) * p.T + s0 + qv : row;
        if (valid) p.lse[li] = (m + log2f(l)) * 0.69314718055994531f;
        const int r0 = q0 + 128 * t + 32 * quarter;  // this warp's first query
        if (!OF32 && !FP8 && r0 < N && (!packed || r0 + 32 <= N)) {
          // bf16 O: each warp stages its 32 rows in its part of the tile's Q
          // buffer (free: the tile's last S MMA has read it) with the 128-byte
          // swizzle and writes them with TMA stores, which clip rows past N.
          // The warp waits only until the stores have read the buffer.
          uint8_t* stg = smem + (t ? L::kQ1 : L::kQ0) + quarter * (32 * D * 2);
          uint8_t* orow = stg + lane * 128;
          const int sw = lane & 7;
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t ov[32];
            tmem_ld32(tO + 32 * c, ov);
            tmem_wait_ld();
#pragma unroll
            for (int x = 0; x < 4; ++x) {
              const int u = 4 * (c & 1) + x;
              *reinterpret_cast<uint4*>(orow + (c >> 1) * 4096 + ((u ^ sw) << 4)) = make_uint4(
                  pack_bf16(__uint_as_float(ov[8 * x + 0]) * inv_l, __uint_as_float(ov[8 * x + 1]) * inv_l),
                  pack_bf16(__uint_as_float(ov[8 * x + 2]) * inv_l, __uint_as_float(ov[8 * x + 3]) * inv_l),
                  pack_bf16(__uint_as_float(ov[8 * x + 4]) * inv_l, __uint_as_float(ov[8 * x + 5]) * inv_l),
                  pack_bf16(__uint_as_float(ov[8 * x + 6]) * inv_l, __uint_as_float(ov[8 * x + 7]) * inv_l));
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
#pragma unroll
            for (int c = 0; c < D / 64; ++c) tma_store_3d(&tm_o, stg + c * 4096, 64 * c, s0 + r0, hq);
            bulk_commit_group();
            if (FA_FWD_STORE_WAIT_READ)
              bulk_wait_group_read0();
            else
              bulk_wait_group0();
          }
          __syncwarp();
        } else {
#pragma unroll
          for (int c = 0; c < D; c += 32) {
            uint32_t ov[32];
            tmem_ld32(tO + c, ov);
            tmem_wait_ld();
            if (valid) {
              if (OF32) {
                float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.o) + row * D + c);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                  dst[e] = make_float4(__uint_as_float(ov[4 * e]) * inv_l, __uint_as_float(ov[4 * e + 1]) * inv_l,
                                       __uint_as_float(ov[4 * e + 2]) * inv_l,
                                       __uint_as_float(ov[4 * e + 3]) * inv_l);
              } else {
                uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.o) + row * D + c);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  uint4 w;
                  w.x = pack_bf16(__uint_as_float(ov[8 * e + 0]) * inv_l, __uint_as_float(ov[8 * e + 1]) * inv_l);
                  w.y = pack_bf16(__uint_as_float(ov[8 * e + 2]) * inv_l, __uint_as_float(ov[8 * e + 3]) * inv_l);
                  w.z = pack_bf16(__uint_as_float(ov[8 * e + 4]) * inv_l, __uint_as_float(ov[8 * e + 5]) * inv_l);
                  w.w = pack_bf16(__uint_as_float(ov[8 * e + 6]) * inv_l, __uint_as_float(ov[8 * e + 7]) * inv_l);
                  dst[e] = w;
                }
              }
            }
          }
        }
      }
    }
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
