// fa_fwd_kernel.cuh -- fused exact-attention forward for sm_100a.
//
// One persistent CTA per SM walks a list of work tiles.  A tile is one
// (batch, query head) and a PAIR of 128-row query blocks; the pair shares one stream
// of 128-key K/V tiles of its key/value head (H / H_kv query heads share one
// key/value head: grouped-query attention, "Flash Attention Explained", "Grouped
// Query Attention"), optionally limited to a causal sliding window (same page,
// "Sliding Window Attention") ("Flash Attention Explained", institutepm.com, "Tile the
// input" / "Fuse into one kernel"; FlashAttention-2's partitioning over the
// sequence dimension, same page, "Flash Attention 1, 2, and 3").
//
// Warp roles (384 threads, three warpgroups):
//   warps 0-3  softmax group 0: one thread per query row of block 0
//   warps 4-7  softmax group 1: one thread per query row of block 1
//   warp  8    TMA producer: Q blocks once per tile, then K_j, V_j into a ring of
//              NSTAGE shared-memory slots (128-byte swizzle)
//   warp  9    MMA issuer: S_i = Q_i K_j^T (both operands in shared memory) and
//              O_i += P_i V_j (P read straight from tensor memory), accumulators
//              in tensor memory; allocates / frees the 512 TMEM columns
//   warps 10-11 idle
// Registers: launched at 168 per thread (384 x 168 = 64512); the softmax warpgroups
// raise theirs to 200 and the producer/MMA warpgroup drops to 104:
// 2 x 128 x 200 + 128 x 104 = 64512.
//
// Tensor memory (512 columns x 128 lanes of 32 bit):
//   [0,128)   S_0  (fp32 scores of block 0; P_0 overwrites its first 64 columns as bf16)
//   [128,256) S_1
//   [256, 256+D)     O_0 (fp32 accumulator)
//   [256+D, 256+2D)  O_1
//
// Per K/V tile the MMA warp issues, in order, PV_0(j), S_0(j+1), PV_1(j), S_1(j+1):
// while one softmax group works on its scores the tensor core computes the other
// group's products (ping-pong).  tcgen05 ops issued by one thread complete in
// order, so S_i(j+1) overwriting P_i(j) is safe, and the commit that signals
// S_i(j+1) also guarantees PV_i(j) has finished.
//
// Online softmax ("Flash Attention Explained", "Compute softmax incrementally";
// holysheep.ai review: running max and sum): scores are taken in base 2,
// x = s * scale * log2(e).  Each row keeps a reference maximum m and a running
// sum l of 2^(x - m).  m is only raised when the tile maximum exceeds it by more
// than TAU (= 8, i.e. a factor 256); then l and the O accumulator are rescaled by
// 2^(m_old - m_new).  Between raises the probabilities stay below 2^TAU, which
// fp32 sums and bf16 P represent without loss, and O / l is unchanged because
// numerator and denominator share the same reference.  Two sums are kept: l of
// the fp32 probabilities (for the log-sum-exp) and lr of the bf16-rounded
// probabilities that actually enter the P.V product, so that O = O_acc / lr is
// an exact convex combination of value rows.  Finally LSE = (m + log2 l) * ln 2.
#pragma once

#include "sm100_ptx.cuh"

namespace fa {

constexpr int kBM = 128;  // query rows per block
constexpr int kBN = 128;  // keys per K/V tile
constexpr int kFwdThreads = 384;
constexpr uint32_t kLaunchRegs = 168;  // 65536 / 384 rounded down to a multiple of 8
constexpr uint32_t kFwdRegsSoftmax = 200;
constexpr uint32_t kFwdRegsOther = 104;
static_assert(2 * 128 * kFwdRegsSoftmax + 128 * kFwdRegsOther <= kFwdThreads * kLaunchRegs,
              "register split exceeds the launch allocation");
// Arrivals that release one P tile: e4m3 rows arrive once per warp (measured 4% faster),
// 16-bit rows once per thread (per-warp arrivals measured 1-3% slower there).
template <Elem E>
constexpr int kPArrivals = E == Elem::kE4M3 ? 4 : 128;
constexpr float kTau = 8.0f;
constexpr float kLn2 = 0.69314718055994530942f;

template <int D, Elem E = Elem::kBf16>
struct FwdCfg {
  static constexpr int kBytes = (E == Elem::kE4M3) ? 1 : 2;    // bytes per element
  static constexpr int kRowBytes = D * kBytes;
  static constexpr int kChunks = kRowBytes / 128;              // 128-byte swizzle chunks per row
  static constexpr int kChunkElems = 128 / kBytes;             // elements per chunk row
  static constexpr int kTileBytes = 128 * kRowBytes;           // one 128-row tile
  static constexpr int kChunkBytes = 128 * 128;                // one 128-row x 128-byte chunk
  static constexpr int kStages = (131072 / kTileBytes) < 16 ? (131072 / kTileBytes) : 16;  // K/V ring slots
  static constexpr int kSSteps = kRowBytes / 32;               // MMA K-steps of S = Q K^T (32 bytes each)
  static constexpr int kPVSteps = kBN * kBytes / 32;           // MMA K-steps of O += P V
  static constexpr int kKeysPerStep = 32 / kBytes;
  static constexpr int kPCols = kBN * kBytes / 4;              // TMEM columns of one P row
  static constexpr uint32_t kOCol = 256;
  static constexpr uint32_t kTmemCols = 512;
  static_assert(kChunks >= 1, "rows of at least 128 bytes");
};

// Output element type: the input type for 16-bit inputs, bf16 for e4m3 inputs.
template <Elem E>
struct FwdOut {
  using T = typename ElemOps<E>::T;
};
template <>
struct FwdOut<Elem::kE4M3> {
  using T = __nv_bfloat16;
};

template <int D, Elem E = Elem::kBf16>
struct __align__(1024) FwdSmem {
  uint8_t q[2][FwdCfg<D, E>::kTileBytes];
  uint8_t kv[FwdCfg<D, E>::kStages][FwdCfg<D, E>::kTileBytes];
  uint64_t q_full[2];
  uint64_t q_empty[2];
  uint64_t kv_full[FwdCfg<D, E>::kStages];
  uint64_t kv_empty[FwdCfg<D, E>::kStages];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_done[2];
  uint64_t mma_drain;
  uint32_t tmem_base;
  int abort_flag;
};

// The k-th tile of CTA c: rounds of G tiles, walked forwards and backwards
// alternately, so heavy and light tiles even out over the rounds.
__device__ __forceinline__ int snake_tile(int c, int k, int G) {
  return k * G + ((k & 1) ? (G - 1 - c) : c);
}

struct FwdTile {
  int b, h, qb0;
};

// Tiles are ordered heaviest first (for causal attention the last query blocks
// see the most keys), heads fastest, so concurrently running CTAs share K/V in L2.
__device__ __forceinline__ FwdTile fwd_decode(int t, int BH, int H, int npairs) {
  FwdTile ti;
  const int p = npairs - 1 - t / BH;
  const int bh = t % BH;
  ti.b = bh / H;
  ti.h = bh % H;
  ti.qb0 = 2 * p;
  return ti;
}

// Key blocks [lo, hi) that query block qb visits (empty past the sequence).  With causal
// masking the last is the diagonal block; with a sliding window of `window` keys before
// the query, the first is the block holding key qb*128 - window.
struct KvRange {
  int lo, hi;
};
template <bool CAUSAL>
__device__ __forceinline__ KvRange fwd_range(int qb, int nkb, int window) {
  KvRange r{0, 0};
  if (qb >= nkb) return r;
  r.hi = CAUSAL ? qb + 1 : nkb;
  if (window >= 0) {
    const int first_key = qb * kBM - window;
    r.lo = first_key > 0 ? first_key / kBN : 0;
  }
  return r;
}

__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity, int* status) {
  // The final wait for issued MMAs, and every wait while unwinding after an abort: ignores
  // the abort flag, still bounded; a timeout here is reported at site 98.
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_test(a, parity)) {
    if (globaltimer_ns() - t0 > FA_WAIT_TIMEOUT_NS) {
      atomicCAS(status, 0, 6 /* FA_ERR_TIMEOUT */);
      atomicCAS(status + 1, 0, 98);
      return false;
    }
  }
  return true;
}

// Probabilities of one score row of NC keys (128 in the prefill kernel): p = 2^(s *
// scale_log2 - m), packed to 16-bit pairs in p[]; adds the fp32 sum to *l and the sum of
// the bf16-rounded values to *lr.
template <Elem E = Elem::kBf16, int NC = kBN>
__device__ __forceinline__ void softmax_row(const uint32_t (&s)[NC], uint32_t (&p)[NC / 2], float scale_log2,
                                            float m, float& l, float& lr) {
  static_assert(E != Elem::kE4M3, "e4m3 rows use softmax_row_e4m3");
  static_assert(NC % 4 == 0, "pairs alternate between two accumulators");
  const float2 sl2 = make_float2(scale_log2, scale_log2);
  const float2 nm2 = make_float2(-m, -m);
  float2 se[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
  float2 sr[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
  for (int c = 0; c < NC / 2; ++c) {
    const float2 x = ffma2(make_float2(__uint_as_float(s[2 * c]), __uint_as_float(s[2 * c + 1])), sl2, nm2);
    const float2 e = make_float2(ex2_approx(x.x), ex2_approx(x.y));
    p[c] = ElemOps<E>::pack(e.x, e.y);
    se[c & 1] = fadd2(se[c & 1], e);
    // the bf16 weights the P.V product actually uses: O = O_acc / lr is an exact
    // convex combination of value rows (the rounding of a dominant weight cancels).
    // fp16 rounds 8x finer, so there lr is the fp32 sum itself.
    if constexpr (E == Elem::kBf16) sr[c & 1] = fadd2(sr[c & 1], ElemOps<E>::unpack(p[c]));
  }
  const float ls = (se[0].x + se[0].y) + (se[1].x + se[1].y);
  l += ls;
  if constexpr (E == Elem::kBf16)
    lr += (sr[0].x + sr[0].y) + (sr[1].x + sr[1].y);
  else
    lr += ls;
}

// e4m3 probabilities of one 128-key score row, four per word (first key in the lowest
// byte); l gets the fp32 sum, lr the sum of the e4m3-rounded values the P.V product uses.
__device__ __forceinline__ void softmax_row_e4m3(const uint32_t (&s)[kBN], uint32_t (&p)[kBN / 4],
                                                 float scale_log2, float m, float& l, float& lr) {
  const float2 sl2 = make_float2(scale_log2, scale_log2);
  const float2 nm2 = make_float2(-m, -m);
  float2 se[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
  float2 sr[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
  for (int c = 0; c < kBN / 4; ++c) {
    const float2 x0 = ffma2(make_float2(__uint_as_float(s[4 * c]), __uint_as_float(s[4 * c + 1])), sl2, nm2);
    const float2 x1 = ffma2(make_float2(__uint_as_float(s[4 * c + 2]), __uint_as_float(s[4 * c + 3])), sl2, nm2);
    const float2 e0 = make_float2(ex2_approx(x0.x), ex2_approx(x0.y));
    const float2 e1 = make_float2(ex2_approx(x1.x), ex2_approx(x1.y));
    p[c] = pack_e4m3x4(e0.x, e0.y, e1.x, e1.y);
    se[c & 1] = fadd2(se[c & 1], fadd2(e0, e1));
    sr[c & 1] = fadd2(sr[c & 1], e4m3x4_pair_sums(p[c]));
  }
  l += (se[0].x + se[0].y) + (se[1].x + se[1].y);
  lr += (sr[0].x + sr[0].y) + (sr[1].x + sr[1].y);
}

template <int D, bool CAUSAL, Elem E = Elem::kBf16>
__global__ void __launch_bounds__(kFwdThreads, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, typename FwdOut<E>::T* __restrict__ out,
                  float* __restrict__ lse, int B, int H, int H_kv, int N, int window, float scale_log2,
                  float out_scale, int* status) {
  using Cfg = FwdCfg<D, E>;
  constexpr int NS = Cfg::kStages;
  extern __shared__ uint8_t smem_raw[];
  FwdSmem<D, E>& sm = *reinterpret_cast<FwdSmem<D, E>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                        ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nkb = (N + kBN - 1) / kBN;
  const int npairs = (nkb + 1) / 2;
  const int BH = B * H;
  const int T = BH * npairs;
  const int group = H / H_kv;  // query heads per key/value head

  if (threadIdx.x == 0) {
    sm.abort_flag = 0;
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.q_full[i], 1);
      mbar_init(&sm.q_empty[i], 1);
      mbar_init(&sm.s_full[i], 1);
      mbar_init(&sm.p_full[i], kPArrivals<E>);
      mbar_init(&sm.o_done[i], 1);
    }
    for (int s = 0; s < NS; ++s) {
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
    }
    mbar_init(&sm.mma_drain, 1);
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(&sm.tmem_base, Cfg::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = sm.tmem_base;

  // Each warpgroup's setmaxnreg sits at the top of the branch holding all of that
  // warpgroup's code, so every instruction after it is compiled within the new limit.
  if (warp >= 8) {
    regs_set<kLaunchRegs, kFwdRegsOther>();
  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const WaitCtx wc{&sm.abort_flag, status, 1};
      uint32_t it = 0, qcnt[2] = {0, 0};
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int t = snake_tile(blockIdx.x, k, gridDim.x);
        if (t >= T) break;
        const FwdTile ti = fwd_decode(t, BH, H, npairs);
        const KvRange rg[2] = {fwd_range<CAUSAL>(ti.qb0, nkb, window), fwd_range<CAUSAL>(ti.qb0 + 1, nkb, window)};
        const int hkv = ti.h / group;
        for (int i = 0; i < 2 && ok; ++i) {
          if (rg[i].hi == rg[i].lo) continue;
          ok = mbar_wait(&sm.q_empty[i], (qcnt[i] & 1) ^ 1, wc);
          if (!ok) break;
          mbar_arrive_expect_tx(&sm.q_full[i], Cfg::kTileBytes);
          for (int c = 0; c < Cfg::kChunks; ++c)
            if (FA_IN_BOUNDS(ti.b < B && ti.h < H && (ti.qb0 + i) * kBM < N && c * Cfg::kChunkElems < D, status, 101))
              tma_load_4d(sm.q[i] + c * Cfg::kChunkBytes, &tm_q, &sm.q_full[i], c * Cfg::kChunkElems, ti.h,
                          (ti.qb0 + i) * kBM, ti.b);
          ++qcnt[i];
        }
        // K/V stream: the union of both blocks' ranges (block 1's range starts and ends later)
        const int jlo = rg[0].lo;
        const int jhi = rg[1].hi > rg[0].hi ? rg[1].hi : rg[0].hi;
        for (int j = jlo; j < jhi && ok; ++j) {
          for (int kv = 0; kv < 2; ++kv, ++it) {
            const int s = it % NS;
            ok = mbar_wait(&sm.kv_empty[s], ((it / NS) & 1) ^ 1, wc);
            if (!ok) break;
            mbar_arrive_expect_tx(&sm.kv_full[s], Cfg::kTileBytes);
            const CUtensorMap* m = kv ? &tm_v : &tm_k;
            for (int c = 0; c < Cfg::kChunks; ++c)
              if (FA_IN_BOUNDS(ti.b < B && hkv < H_kv && j >= 0 && j * kBN < N && c * Cfg::kChunkElems < D, status,
                               102))
                tma_load_4d(sm.kv[s] + c * Cfg::kChunkBytes, m, &sm.kv_full[s], c * Cfg::kChunkElems, hkv,
                            j * kBN, ti.b);
          }
        }
      }
      if (!ok) {
        // Unwinding: wait (bounded) for the copies still in flight before the CTA exits.
        for (uint32_t idx = (it > (uint32_t)NS ? it - NS : 0); idx < it; ++idx)
          mbar_wait_drain(&sm.kv_full[idx % NS], (idx / NS) & 1, status);
        for (int i = 0; i < 2; ++i)
          if (qcnt[i] > 0) mbar_wait_drain(&sm.q_full[i], (qcnt[i] - 1) & 1, status);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    {  // the whole warp walks the issuer's path; one elected lane issues each MMA and commit
      const WaitCtx wc{&sm.abort_flag, status, 2};
      constexpr uint32_t idesc_s = idesc_kind_f16(128, kBN, 0, 0, ElemOps<E>::kMmaType);  // Q, K K-major
      constexpr uint32_t idesc_o = idesc_kind_f16(128, D, 0, 1, ElemOps<E>::kMmaType);    // P in TMEM, V MN-major
      const uint32_t q_addr[2] = {smem_u32(sm.q[0]), smem_u32(sm.q[1])};
      const uint32_t kv_addr0 = smem_u32(sm.kv[0]);
      uint32_t it = 0, qcnt[2] = {0, 0}, pcnt[2] = {0, 0};
      bool ok = true;

      // Descriptors differ only in the start-address field (low 14 bits, 16-byte units),
      // so each MMA adds an offset to one base descriptor.
      const uint64_t dq[2] = {sdesc_sw128(q_addr[0], 16, 1024), sdesc_sw128(q_addr[1], 16, 1024)};
      const uint64_t dk0 = sdesc_sw128(kv_addr0, 16, 1024);
      const uint64_t dv0 = sdesc_sw128(kv_addr0, Cfg::kChunkBytes, 1024);
      auto issue_s = [&](int i, int slot) {
        const uint32_t tS = tbase + i * 128;
        const uint64_t dk = dk0 + static_cast<uint64_t>((slot * Cfg::kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < Cfg::kSSteps; ++kk) {
          const uint32_t off = ((kk / 4) * Cfg::kChunkBytes + (kk % 4) * 32) >> 4;
          if constexpr (E == Elem::kE4M3)
            umma_ss_f8_w(tS, dq[i] + off, dk + off, idesc_s, kk > 0);
          else
            umma_ss_w(tS, dq[i] + off, dk + off, idesc_s, kk > 0);
        }
      };
      auto issue_pv = [&](int i, int slot, uint32_t acc) {
        const uint32_t tO = tbase + Cfg::kOCol + i * D;
        const uint32_t tP = tbase + i * 128;
        const uint64_t dv = dv0 + static_cast<uint64_t>((slot * Cfg::kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < Cfg::kPVSteps; ++kk) {
          if constexpr (E == Elem::kE4M3)
            umma_ts_f8_w(tO, tP + kk * 8, dv + ((kk * Cfg::kKeysPerStep * 128) >> 4), idesc_o, (kk > 0) || acc);
          else
            umma_ts_w(tO, tP + kk * 8, dv + ((kk * Cfg::kKeysPerStep * 128) >> 4), idesc_o, (kk > 0) || acc);
        }
      };

      for (int k = 0; ok; ++k) {
        const int t = snake_tile(blockIdx.x, k, gridDim.x);
        if (t >= T) break;
        const FwdTile ti = fwd_decode(t, BH, H, npairs);
        const KvRange rg[2] = {fwd_range<CAUSAL>(ti.qb0, nkb, window), fwd_range<CAUSAL>(ti.qb0 + 1, nkb, window)};
        const int jlo = rg[0].lo;
        const int jhi = rg[1].hi > rg[0].hi ? rg[1].hi : rg[0].hi;
        auto in = [&](int i, int j) { return j >= rg[i].lo && j < rg[i].hi; };
        for (int i = 0; i < 2 && ok; ++i)
          if (rg[i].hi > rg[i].lo) ok = __all_sync(0xffffffffu, mbar_wait(&sm.q_full[i], qcnt[i] & 1, wc));
        if (!ok) break;
        // prologue: S_i for the first key block
        const int sk0 = it % NS;
        ok = __all_sync(0xffffffffu, mbar_wait(&sm.kv_full[sk0], (it / NS) & 1, wc));
        if (!ok) break;
        ++it;
        tc_fence_after();
        for (int i = 0; i < 2; ++i) {
          if (!in(i, jlo)) continue;
          issue_s(i, sk0);
          umma_commit_w(&sm.s_full[i]);
          if (rg[i].hi == jlo + 1) umma_commit_w(&sm.q_empty[i]);
        }
        umma_commit_w(&sm.kv_empty[sk0]);
        for (int j = jlo; j < jhi && ok; ++j) {
          const int sv = it % NS;
          ok = __all_sync(0xffffffffu, mbar_wait(&sm.kv_full[sv], (it / NS) & 1, wc));
          if (!ok) break;
          ++it;
          int skn = -1;
          if (j + 1 < jhi) {
            skn = it % NS;
            ok = __all_sync(0xffffffffu, mbar_wait(&sm.kv_full[skn], (it / NS) & 1, wc));
            if (!ok) break;
            ++it;
          }
          for (int i = 0; i < 2 && ok; ++i) {
            if (in(i, j)) {
              ok = __all_sync(0xffffffffu, mbar_wait(&sm.p_full[i], pcnt[i] & 1, wc));
              if (!ok) break;
              ++pcnt[i];
              tc_fence_after();
              issue_pv(i, sv, j > rg[i].lo);
              if (j + 1 == rg[i].hi) umma_commit_w(&sm.o_done[i]);
            }
            if (in(i, j + 1)) {
              issue_s(i, skn);
              umma_commit_w(&sm.s_full[i]);
              if (j + 2 == rg[i].hi) umma_commit_w(&sm.q_empty[i]);
            }
          }
          if (!ok) break;
          umma_commit_w(&sm.kv_empty[sv]);
          if (skn >= 0) umma_commit_w(&sm.kv_empty[skn]);
        }
        for (int i = 0; i < 2; ++i)
          if (rg[i].hi > rg[i].lo) ++qcnt[i];
      }
      // Wait for every MMA issued to finish before the columns are freed.
      umma_commit_w(&sm.mma_drain);
      mbar_wait_drain(&sm.mma_drain, 0, status);
    }
    __syncwarp();
  }
  } else {
    // ------------------------------------------------------------ softmax groups
    regs_set<kLaunchRegs, kFwdRegsSoftmax>();
    const int g = warp >> 2;             // which query block of the pair
    const int r = threadIdx.x & 127;     // row within the block == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tbase + g * 128 + lane_off;
    const uint32_t tO = tbase + Cfg::kOCol + g * D + lane_off;
    const WaitCtx wc{&sm.abort_flag, status, 3 + g};
    uint32_t scnt = 0, ocnt = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int t = snake_tile(blockIdx.x, k, gridDim.x);
      if (t >= T) break;
      const FwdTile ti = fwd_decode(t, BH, H, npairs);
      const int qb = ti.qb0 + g;
      const KvRange rg = fwd_range<CAUSAL>(qb, nkb, window);
      if (rg.hi == rg.lo) continue;
      const int row = qb * kBM + r;
      float m_ref = -INFINITY;
      float l = 0.f;    // sum of 2^(x - m) in fp32: the log-sum-exp
      float lr = 0.f;   // sum of the same weights rounded to bf16: normalises O
      for (int j = rg.lo; j < rg.hi; ++j) {
        ok = __all_sync(0xffffffffu, mbar_wait(&sm.s_full[g], scnt & 1, wc));
        if (!ok) break;
        ++scnt;
        tc_fence_after();
        uint32_t s[kBN];
        tmem_ld32(tS + 0, s + 0);
        tmem_ld32(tS + 32, s + 32);
        tmem_ld32(tS + 64, s + 64);
        tmem_ld32(tS + 96, s + 96);
        tmem_wait_ld();
        const int k0 = j * kBN;
        // masking: the diagonal / last tile (causal, or keys past N), and with a window the
        // tiles that start before some row's first visible key
        const bool edge = window >= 0 && k0 < qb * kBM + kBM - 1 - window;
        const bool masked = ((j == rg.hi - 1) && (CAUSAL || (N % kBN) != 0)) || edge;
        if (masked) {
          int lim = N - 1 - k0;                    // last valid key column of this tile
          if (CAUSAL) lim = min(lim, row - k0);    // key <= query
          const int first = window >= 0 ? row - window - k0 : 0;  // key >= query - window
#pragma unroll
          for (int c = 0; c < kBN; ++c)
            if (c > lim || c < first) s[c] = __float_as_uint(-INFINITY);
        }
        // row maximum: 8 independent chains of three-input max, then combine
        float mx8[8];
#pragma unroll
        for (int x = 0; x < 8; ++x) mx8[x] = fmaxf(__uint_as_float(s[x]), __uint_as_float(s[x + 8]));
#pragma unroll
        for (int c = 16; c < kBN; c += 16)
#pragma unroll
          for (int x = 0; x < 8; ++x)
            mx8[x] = fmax3(mx8[x], __uint_as_float(s[c + x]), __uint_as_float(s[c + 8 + x]));
        const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                               fmaxf(mx8[6], mx8[7]));
        const float m_new = mx * scale_log2;
        const bool raise = m_new > m_ref + kTau;
        if (__any_sync(0xffffffffu, raise)) {
          const float alpha = raise ? ex2_approx(m_ref - m_new) : 1.0f;
          if (raise) {
            l *= alpha;
            lr *= alpha;
            m_ref = m_new;
          }
          if (j > rg.lo) {
            // PV(j-1) is complete: the commit that signalled S(j) covers it.
#pragma unroll 1
            for (int c = 0; c < D; c += 32) {
              uint32_t o[32];
              tmem_ld32(tO + c, o);
              tmem_wait_ld();
#pragma unroll
              for (int x = 0; x < 32; ++x) o[x] = __float_as_uint(__uint_as_float(o[x]) * alpha);
              tmem_st32(tO + c, o);
            }
            tmem_wait_st();
          }
        }
        uint32_t p[Cfg::kPCols];
        // a row that has seen no visible key yet (window edge) keeps m = -inf; use 0 as its
        // reference so that 2^(-inf - m) stays 0 instead of NaN
        const float m_use = m_ref == -INFINITY ? 0.f : m_ref;
        // masked scores are -inf, and ex2 of -inf is exactly 0
        if constexpr (E == Elem::kE4M3) {
          softmax_row_e4m3(s, p, scale_log2, m_use, l, lr);
          tmem_st32(tS + 0, p);
        } else {
          softmax_row<E>(s, p, scale_log2, m_use, l, lr);
          tmem_st32(tS + 0, p);
          tmem_st32(tS + 32, p + 32);
        }
        tmem_wait_st();
        tc_fence_before();
        if constexpr (kPArrivals<E> == 4) {
          __syncwarp();
          if ((r & 31) == 0) mbar_arrive(&sm.p_full[g]);
        } else {
          mbar_arrive(&sm.p_full[g]);
        }
      }
      if (!ok) break;
      // epilogue: O = O_acc / l, LSE = (m + log2 l) ln 2
      ok = __all_sync(0xffffffffu, mbar_wait(&sm.o_done[g], ocnt & 1, wc));
      if (!ok) break;
      ++ocnt;
      tc_fence_after();
      // e4m3 inputs: out_scale is V's dequantisation factor
      const float inv_l = (E == Elem::kE4M3 ? out_scale : 1.0f) / lr;
      const bool live = row < N;
      typename FwdOut<E>::T* orow = out + ((static_cast<int64_t>(ti.b) * N + row) * H + ti.h) * D;
#pragma unroll 1
      for (int c = 0; c < D; c += 32) {
        uint32_t o[32];
        tmem_ld32(tO + c, o);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int x = 0; x < 16; ++x)
          pk[x] = ElemOps<E == Elem::kE4M3 ? Elem::kBf16 : E>::pack(__uint_as_float(o[2 * x]) * inv_l,
                                                                   __uint_as_float(o[2 * x + 1]) * inv_l);
        if (live && FA_IN_BOUNDS(((static_cast<int64_t>(ti.b) * N + row) * H + ti.h) * D + c + 32 <=
                                     static_cast<int64_t>(B) * N * H * D && ti.h < H && row >= 0,
                                 status, 103)) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c);
#pragma unroll
          for (int x = 0; x < 4; ++x) dst[x] = make_uint4(pk[4 * x], pk[4 * x + 1], pk[4 * x + 2], pk[4 * x + 3]);
        }
      }
      if (live && FA_IN_BOUNDS((static_cast<int64_t>(ti.b) * H + ti.h) * N + row < static_cast<int64_t>(B) * H * N,
                               status, 104))
        lse[(static_cast<int64_t>(ti.b) * H + ti.h) * N + row] = (m_ref + lg2_approx(l)) * kLn2;
      tc_fence_before();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tbase, Cfg::kTmemCols);
  }
}

}  // namespace fa
