// fa_decode_kernel.cuh -- split-KV exact attention of a few new queries per sequence
// against a key/value cache (decoding), for sm_100a.
//
// In the generation phase each sequence adds one (or a few) query rows while its keys
// and values come from the cache of everything before them ("What Is Flash Attention?",
// bestllmfor.com, table "What you actually gain on a local machine": prompt processing
// vs token generation).  Nothing is reused across queries, so the kernel is a stream over
// the cache and is sized for HBM bandwidth.
//
// Work list.  The unit is one 128-key tile of one (sequence b, key/value head) PAIR.  The
// tiles of all pairs are laid end to end (pairs ordered b-major) and CTA c of the
// persistent grid takes tiles [c*L, (c+1)*L), L = ceil(total / grid), so every CTA
// streams the same number of tiles whatever the mix of cache lengths.  The lengths are
// read on the device (seqlens), so the schedule needs no host round trip.  A CTA's run
// falls into SEGMENTS, each inside one pair.
//
// Rows.  The G = H / H_kv query heads that share a key/value head and the N_q new
// positions form the rows r = i*G + g of a tile ("Flash Attention Explained",
// institutepm.com, "Grouped Query Attention"): the tile's K/V stream is read once for
// all of them.  Up to 64 rows use M = 64 MMAs, whose accumulators occupy lanes 0-15 of
// each 32-lane quarter of tensor memory (half the tensor work of M = 128, which only
// larger groups use).  The rows are copied to fill the tile: with M = G*N_q <= 16 (or
// <= 32) rows, R = 4 (or 2) copies, copy c in quarters [c*4/R, (c+1)*4/R); copy c takes
// keys [c*128/R, (c+1)*128/R) of every tile, so each softmax warp handles 128/R keys per
// tile instead of 128.  The copies are independent online softmaxes over disjoint key
// subsets, merged like any other partial results.  Lanes past a copy's rows are padding
// and are never written out.
//
// Two key streams.  The even tiles of a segment go to stream 0 and the odd tiles to
// stream 1, each with its own score buffer, accumulator and row state, so the tensor core
// always has two independent chains: while the softmax warps work on one stream's scores
// it runs the other stream's products.  Each stream runs the prefill kernel's online
// softmax (running maximum with conditional rescale, fp32 sum l for the LSE, bf16-rounded
// sum lr for O).  At the end of a segment each thread merges its row's two streams with
// log-sum-exp weights and writes the result: the final O and LSE when the segment is the
// whole pair and R = 1, otherwise an fp32 partial per copy (O normalised, plus the
// natural-log sums of l and of lr) that fa_decode_merge_kernel combines.
//
// Stale cache.  Keys at or past a sequence's length are masked.  The value rows of a
// tile past the length are zeroed in shared memory before the P.V product: a zero
// weight times a stale NaN would still be NaN.
//
// Warp roles (192 threads, so up to 255 registers each): warps 0-3 softmax of both streams
// (one thread per tile row; only the warps holding real rows take part),
// warp 4 TMA producer, warp 5 MMA issuer.  The cache stream, not the softmax, bounds the
// kernel: at full HBM bandwidth one SM has ~2800 cycles per 128-key tile.
//
// Tensor memory (512 columns): [0,128) S_0, [128,256) S_1 (P_i overwrites the first 64
// columns of S_i as bf16), [256, 256+D) O_0, [256+D, 256+2D) O_1.
#pragma once

#include "fa_fwd_kernel.cuh"

namespace fa {

constexpr int kDecThreads = 192;
constexpr int kDecMaxRows = 128;  // G * N_q rows per tile

template <int D>
struct DecCfg {
  static constexpr int kChunks = D / 64;
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kChunkBytes = 128 * 128;
#ifdef FA_DEC_STAGES
  static constexpr int kStages = FA_DEC_STAGES * (128 / D);
#else
  static constexpr int kStages = (D == 128) ? 4 : 8;  // K/V ring slots
#endif
  static constexpr uint32_t kOCol = 256;
  static constexpr uint32_t kTmemCols = 512;
};

// This CTA's slice of the flattened tile list: tiles [t0, t1), the first of them inside
// pair p0, whose first tile has flattened index start0.
struct DecPlan {
  int t0, t1, p0, start0;
};

template <int D>
struct __align__(1024) DecSmem {
  uint8_t q[2][DecCfg<D>::kTileBytes];
  uint8_t kv[DecCfg<D>::kStages][DecCfg<D>::kTileBytes];
  uint64_t q_full[2];
  uint64_t q_empty[2];
  uint64_t kv_full[DecCfg<D>::kStages];
  uint64_t kv_empty[DecCfg<D>::kStages];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_done[2];
  uint64_t mma_drain;
  DecPlan plan;
  uint32_t tmem_base;
  int abort_flag;
};

// MMA rows for M real rows (64 when they fit, else 128) and row copies per tile: 4 when
// M <= 16, 2 when M <= 32, else 1.
__host__ __device__ constexpr int dec_mma_rows(int M) { return M <= 64 ? 64 : 128; }
__host__ __device__ constexpr int dec_copies(int M) { return M <= 16 ? 4 : (M <= 32 ? 2 : 1); }

struct DecArgs {
  const int* seqlens;      // [B] cached length of each sequence, or null: all N_kv
  void* out;               // [B, N_q, H, D], bf16 or fp16
  float* lse;              // [B, H, N_q]
  int* meta;               // [2 + B]: total tiles, tiles per CTA, per-sequence tile prefix
  float* part_lse;         // [slots * R, M, 2]: natural-log sums of l and of lr of a segment
  float* part_o;           // [slots * R, M, D]: segment output, normalised by its lr
  int B, H, H_kv, N_q, N_kv, window, causal;
  int R;                   // row copies per tile (dec_copies of M)
  float scale_log2;
  long long slots;         // partial slots in part_lse / part_o (for the checking build)
  int* status;             // device status word (the merge kernel's bounds checks)
};

// Cached length of sequence b (clamped to the capacity), the first key tile any of its
// queries can see, and its number of key tiles.
struct DecSeq {
  int len, kt_lo, T;
};
__device__ __forceinline__ DecSeq dec_seq(const DecArgs& a, int b) {
  int len = a.seqlens ? __ldg(a.seqlens + b) : a.N_kv;
  len = min(max(len, 0), a.N_kv);
  DecSeq s;
  s.len = len;
  s.kt_lo = (a.causal && a.window >= 0) ? max(0, len - a.N_q - a.window) / 128 : 0;
  s.T = len > 0 ? (len + 127) / 128 - s.kt_lo : 0;
  return s;
}

// One warp: the total tile count, this CTA's slice and the pair it starts in.  With
// write_meta the warp also stores the per-sequence prefix for the merge kernel.
__device__ __forceinline__ void dec_plan(const DecArgs& a, int lane, DecPlan* out, bool write_meta) {
  constexpr unsigned kFull = 0xffffffffu;
  int total = 0;
  for (int b0 = 0; b0 < a.B; b0 += 32) {
    const int b = b0 + lane;
    const int v = b < a.B ? dec_seq(a, b).T * a.H_kv : 0;
    total += static_cast<int>(__reduce_add_sync(kFull, static_cast<unsigned>(v)));
  }
  const int per = total > 0 ? (total + static_cast<int>(gridDim.x) - 1) / static_cast<int>(gridDim.x) : 1;
  const int t0 = min(total, static_cast<int>(blockIdx.x) * per);
  const int t1 = min(total, t0 + per);
  int p0 = 0, start0 = 0;
  bool found = t0 >= t1;
  int acc = 0;
  for (int b0 = 0; b0 < a.B && (!found || write_meta); b0 += 32) {
    const int b = b0 + lane;
    const int T = b < a.B ? dec_seq(a, b).T : 0;
    const int v = T * a.H_kv;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(kFull, incl, o);
      if (lane >= o) incl += y;
    }
    incl += acc;
    const int excl = incl - v;
    if (write_meta && b < a.B) a.meta[2 + b] = excl;
    const unsigned hit = __ballot_sync(kFull, !found && b < a.B && excl <= t0 && t0 < incl);
    if (hit) {
      const int src = __ffs(hit) - 1;
      const int e = __shfl_sync(kFull, excl, src);
      const int tb = __shfl_sync(kFull, T, src);
      const int kvh = (t0 - e) / tb;
      p0 = (b0 + src) * a.H_kv + kvh;
      start0 = e + kvh * tb;
      found = true;
    }
    acc = __shfl_sync(kFull, incl, 31);
  }
  if (lane == 0) {
    if (write_meta) {
      a.meta[0] = total;
      a.meta[1] = per;
    }
    out->t0 = t0;
    out->t1 = t1;
    out->p0 = p0;
    out->start0 = start0;
  }
}

// A run of n consecutive key tiles of pair p = (b, kvh), starting at absolute tile kt0.
struct DecSeg {
  int p, b, kvh, len, kt0, n;
  bool whole;  // the run is the whole pair: write the final output directly
};

// Walks this CTA's slice segment by segment; every role walks it the same way.
struct DecWalk {
  int t, t1, p, pstart;
  __device__ __forceinline__ explicit DecWalk(const DecPlan& pl) : t(pl.t0), t1(pl.t1), p(pl.p0), pstart(pl.start0) {}
  __device__ __forceinline__ bool next(const DecArgs& a, DecSeg& s) {
    if (t >= t1) return false;
    DecSeq q = dec_seq(a, p / a.H_kv);
    while (t >= pstart + q.T) {  // finished (or empty) pairs; t < t1 <= total keeps p in range
      pstart += q.T;
      ++p;
      q = dec_seq(a, p / a.H_kv);
    }
    const int end = min(pstart + q.T, t1);
    s.p = p;
    s.b = p / a.H_kv;
    s.kvh = p - s.b * a.H_kv;
    s.len = q.len;
    s.kt0 = q.kt_lo + (t - pstart);
    s.n = end - t;
    s.whole = (t == pstart) && (end == pstart + q.T);
    t = end;
    return true;
  }
};

template <int D, Elem E = Elem::kBf16, int R = 1, int kM = 128>
__global__ void __launch_bounds__(kDecThreads, 1)
    fa_decode_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const DecArgs a, int* status) {
  using Cfg = DecCfg<D>;
  constexpr int NS = Cfg::kStages;
  constexpr unsigned kFull = 0xffffffffu;
  extern __shared__ uint8_t smem_raw[];
  DecSmem<D>& sm = *reinterpret_cast<DecSmem<D>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                  ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = a.H / a.H_kv;
  const int M = G * a.N_q;              // real rows of a copy (<= kM / R)
  static_assert(kM == 64 || kM == 128, "tcgen05 M of one CTA");
  constexpr int kQuarterRows = kM / 4;     // accumulator lanes used per 32-lane quarter
  constexpr int kWarpsPerCopy = 4 / R;
  constexpr int kCopyRows = kM / R;        // tile rows per copy
  constexpr int kCopyKeys = 128 / R;       // keys per copy in a tile
  // softmax warps holding real rows: the first ceil(M / kQuarterRows) warps of every copy
  const int aw = ((M + kQuarterRows - 1) / kQuarterRows) * R;

  if (threadIdx.x == 0) {
    sm.abort_flag = 0;
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.q_full[i], 1);
      mbar_init(&sm.q_empty[i], 1);
      mbar_init(&sm.s_full[i], 1);
      mbar_init(&sm.p_full[i], 32 * aw);
      mbar_init(&sm.o_done[i], 1);
    }
    for (int s = 0; s < NS; ++s) {
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
    }
    mbar_init(&sm.mma_drain, 1);
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(&sm.tmem_base, Cfg::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 4) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
    }
    dec_plan(a, lane, &sm.plan, blockIdx.x == 0);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = sm.tmem_base;
  const DecPlan plan = sm.plan;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const WaitCtx wc{&sm.abort_flag, status, 21};
      DecWalk w(plan);
      DecSeg s;
      uint32_t it = 0, qc = 0;
      bool ok = true;
      while (ok && w.next(a, s)) {
        const int qi = qc & 1;
        ok = mbar_wait(&sm.q_empty[qi], ((qc >> 1) & 1) ^ 1, wc);
        if (!ok) break;
        // the G heads x N_q positions of this key/value head: one box per 64-column chunk
        // and row copy (copy c at row c * 128 / R; a multiple of 8 rows keeps the swizzle)
        mbar_arrive_expect_tx(&sm.q_full[qi], static_cast<uint32_t>(R * Cfg::kChunks * 128 * M));
        for (int cp = 0; cp < R; ++cp)
          for (int c = 0; c < Cfg::kChunks; ++c)
            if (FA_IN_BOUNDS(s.b < a.B && s.kvh * G + G <= a.H && c * 64 < D, status, 301))
              tma_load_4d(sm.q[qi] + c * Cfg::kChunkBytes + cp * kCopyRows * 128, &tm_q, &sm.q_full[qi], c * 64,
                          s.kvh * G, 0, s.b);
        ++qc;
        // K/V tiles in the order the MMA warp consumes them: K0, K1, then V_t, K_{t+2}
        auto load = [&](const CUtensorMap* m, int t) -> bool {
          const int slot = it % NS;
          if (!mbar_wait(&sm.kv_empty[slot], ((it / NS) & 1) ^ 1, wc)) return false;
          mbar_arrive_expect_tx(&sm.kv_full[slot], Cfg::kTileBytes);
          for (int c = 0; c < Cfg::kChunks; ++c)
            if (FA_IN_BOUNDS(s.b < a.B && s.kvh < a.H_kv && s.kt0 + t >= 0 && (s.kt0 + t) * 128 < a.N_kv, status, 302))
              tma_load_4d(sm.kv[slot] + c * Cfg::kChunkBytes, m, &sm.kv_full[slot], c * 64, s.kvh,
                          (s.kt0 + t) * 128, s.b);
          ++it;
          return true;
        };
        ok = load(&tm_k, 0) && (s.n < 2 || load(&tm_k, 1));
        for (int t = 0; t < s.n && ok; ++t) ok = load(&tm_v, t) && (t + 2 >= s.n || load(&tm_k, t + 2));
      }
      if (!ok) {
        // Unwinding: wait (bounded) for the copies still in flight before the CTA exits.
        for (uint32_t idx = (it > static_cast<uint32_t>(NS) ? it - NS : 0); idx < it; ++idx)
          mbar_wait_drain(&sm.kv_full[idx % NS], (idx / NS) & 1, status);
        for (uint32_t u = (qc > 2 ? qc - 2 : 0); u < qc; ++u) mbar_wait_drain(&sm.q_full[u & 1], (u >> 1) & 1, status);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer (the whole warp
    // waits and zeroes stale value rows; one elected lane issues each MMA and commit)
    const WaitCtx wc{&sm.abort_flag, status, 22};
    constexpr uint32_t idesc_s = idesc_kind_f16(kM, kBN, 0, 0, ElemOps<E>::kMmaType);  // Q, K K-major
    constexpr uint32_t idesc_o = idesc_kind_f16(kM, D, 0, 1, ElemOps<E>::kMmaType);    // P in TMEM, V MN-major
    const uint32_t kv_addr0 = smem_u32(sm.kv[0]);
    const uint64_t dq0 = sdesc_sw128(smem_u32(sm.q[0]), 16, 1024);
    const uint64_t dq1 = sdesc_sw128(smem_u32(sm.q[1]), 16, 1024);
    const uint64_t dk0 = sdesc_sw128(kv_addr0, 16, 1024);
    const uint64_t dv0 = sdesc_sw128(kv_addr0, Cfg::kChunkBytes, 1024);
    auto issue_s = [&](int i, int qi, int slot) {
      const uint32_t tS = tbase + i * 128;
      const uint64_t dk = dk0 + static_cast<uint64_t>((slot * Cfg::kTileBytes) >> 4);
      const uint64_t dq = qi ? dq1 : dq0;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = ((kk / 4) * Cfg::kChunkBytes + (kk % 4) * 32) >> 4;
        umma_ss_w(tS, dq + off, dk + off, idesc_s, kk > 0);
      }
    };
    auto issue_pv = [&](int i, int slot, uint32_t acc) {
      const uint32_t tO = tbase + Cfg::kOCol + i * D;
      const uint32_t tP = tbase + i * 128;
      const uint64_t dv = dv0 + static_cast<uint64_t>((slot * Cfg::kTileBytes) >> 4);
#pragma unroll
      for (int kk = 0; kk < kBN / 16; ++kk)
        umma_ts_w(tO, tP + kk * 8, dv + ((kk * 16 * 128) >> 4), idesc_o, (kk > 0) || acc);
    };
    auto wait_all = [&](uint64_t* bar, uint32_t parity) { return __all_sync(kFull, mbar_wait(bar, parity, wc)); };

    DecWalk w(plan);
    DecSeg s;
    uint32_t it = 0, qc = 0, pcnt0 = 0, pcnt1 = 0;  // P hand-offs consumed per stream
    bool ok = true;
    int slot = 0;
    auto take = [&]() -> bool {
      slot = it % NS;
      const bool r = wait_all(&sm.kv_full[slot], (it / NS) & 1);
      ++it;
      return r;
    };
    while (ok && w.next(a, s)) {
      const int qi = qc & 1;
      ok = wait_all(&sm.q_full[qi], (qc >> 1) & 1);
      if (!ok) break;
      ++qc;
      tc_fence_after();
      for (int t = 0; t < 2 && t < s.n && ok; ++t) {
        ok = take();
        if (!ok) break;
        tc_fence_after();
        issue_s(t, qi, slot);
        umma_commit_w(&sm.s_full[t]);
        umma_commit_w(&sm.kv_empty[slot]);
        if (t == s.n - 1) umma_commit_w(&sm.q_empty[qi]);
      }
      for (int t = 0; t < s.n && ok; ++t) {
        const int i = t & 1;
        ok = wait_all(&sm.p_full[i], (i ? pcnt1 : pcnt0) & 1);
        if (!ok) break;
        if (i) ++pcnt1; else ++pcnt0;
        ok = take();  // V_t
        if (!ok) break;
        // rows [z0, z1) of this value tile lie past the sequence but inside the cache:
        // stale slots, zeroed so that their zero weights give exact zeros
        const int kb = (s.kt0 + t) * 128;
        const int z0 = s.len - kb;
        const int z1 = min(128, a.N_kv - kb);
        if (z0 < z1) {
          constexpr int kUnits = Cfg::kChunks * 8;  // 16-byte units per row
          for (int u = lane; u < (z1 - z0) * kUnits; u += 32) {
            const int row = z0 + u / kUnits;
            const int rem = u % kUnits;
            *reinterpret_cast<uint4*>(sm.kv[slot] + (rem / 8) * Cfg::kChunkBytes + row * 128 + (rem % 8) * 16) =
                make_uint4(0u, 0u, 0u, 0u);
          }
          fence_proxy_async_smem();
          __syncwarp();
        }
        tc_fence_after();
        issue_pv(i, slot, t >= 2);
        umma_commit_w(&sm.kv_empty[slot]);
        if (t + 2 >= s.n) umma_commit_w(&sm.o_done[i]);
        if (t + 2 < s.n) {
          ok = take();  // K_{t+2}
          if (!ok) break;
          tc_fence_after();
          issue_s(i, qi, slot);
          umma_commit_w(&sm.s_full[i]);
          umma_commit_w(&sm.kv_empty[slot]);
          if (t + 2 == s.n - 1) umma_commit_w(&sm.q_empty[qi]);
        }
      }
    }
    // Wait for every MMA issued to finish before the columns are freed.
    umma_commit_w(&sm.mma_drain);
    mbar_wait_drain(&sm.mma_drain, 0, status);
    __syncwarp();
  } else if (warp < 4 && (warp % kWarpsPerCopy) * kQuarterRows < M) {
    // ------------------------------------------------------------ softmax, both streams
    constexpr int NC = kCopyKeys;                 // keys of a tile this warp handles
    const int cp = warp / kWarpsPerCopy;          // row copy
    const int col0 = cp * NC;                     // its first key column in the tile
    // row within the copy; with M = 64 lanes 16-31 of the quarter hold no accumulator rows
    const int rc = lane < kQuarterRows ? (warp % kWarpsPerCopy) * kQuarterRows + lane : 1 << 20;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t tS0 = tbase + lane_off;                 // stream i: + i * 128
    const uint32_t tO0 = tbase + Cfg::kOCol + lane_off;    // stream i: + i * D
    const WaitCtx wc{&sm.abort_flag, status, 23};
    uint32_t zero[16];
#pragma unroll
    for (int x = 0; x < 16; ++x) zero[x] = 0u;
    DecWalk w(plan);
    DecSeg s;
    uint32_t scnt0 = 0, scnt1 = 0, ocnt0 = 0, ocnt1 = 0;
    bool ok = true;
    while (ok && w.next(a, s)) {
      // row state of the stream the next tile belongs to (c) and of the other one (x);
      // swapped after every tile, since the tiles alternate between the streams
      float mc = -INFINITY, lc = 0.f, lrc = 0.f;
      float mx_ = -INFINITY, lx = 0.f, lrx = 0.f;
      for (int t = 0; t < s.n; ++t) {
        const int i = t & 1;
        const int k0 = (s.kt0 + t) * kBN + col0;    // this copy's first key
        const uint32_t tS = tS0 + i * 128;
        const uint32_t tO = tO0 + i * D;
        ok = __all_sync(kFull, mbar_wait(&sm.s_full[i], (i ? scnt1 : scnt0) & 1, wc));
        if (!ok) break;
        if (i) ++scnt1; else ++scnt0;
        tc_fence_after();
        uint32_t sv[NC];
#pragma unroll
        for (int c = 0; c < NC; c += 32) tmem_ld32(tS + col0 + c, sv + c);
        tmem_wait_ld();
        // every real row sees the keys up to all_hi and from all_lo on
        const int all_hi = a.causal ? s.len - a.N_q : s.len - 1;
        const int all_lo = a.window >= 0 ? s.len - 1 - a.window : 0;
        const bool masked = (k0 + NC - 1 > all_hi) || (k0 < all_lo);
        if (masked) {
          // this row's visible keys: [vis_lo, vis_hi]
          const int qpos = s.len - a.N_q + rc / G;
          const int vis_hi = rc >= M ? -1 : (a.causal ? qpos : s.len - 1);
          const int vis_lo = a.window >= 0 ? qpos - a.window : 0;
          const int lim = vis_hi - k0;
          const int first = vis_lo - k0;
#pragma unroll
          for (int c = 0; c < NC; ++c)
            if (c > lim || c < first) sv[c] = __float_as_uint(-INFINITY);
        }
        float mx8[8];
#pragma unroll
        for (int x = 0; x < 8; ++x) mx8[x] = fmaxf(__uint_as_float(sv[x]), __uint_as_float(sv[x + 8]));
#pragma unroll
        for (int c = 16; c < NC; c += 16)
#pragma unroll
          for (int x = 0; x < 8; ++x)
            mx8[x] = fmax3(mx8[x], __uint_as_float(sv[c + x]), __uint_as_float(sv[c + 8 + x]));
        const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                               fmaxf(mx8[6], mx8[7]));
        const float m_new = mx * a.scale_log2;
        const bool raise = m_new > mc + kTau;
        if (__any_sync(kFull, raise)) {
          const float alpha = raise ? ex2_approx(mc - m_new) : 1.0f;
          if (raise) {
            lc *= alpha;
            lrc *= alpha;
            mc = m_new;
          }
          if (t >= 2) {
            // this stream's previous P.V is complete: the commit that signalled this S
            // was issued after it
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
        uint32_t p[NC / 2];
        const float m_use = mc == -INFINITY ? 0.f : mc;
        softmax_row<E, NC>(sv, p, a.scale_log2, m_use, lc, lrc);
        // P for all 128 keys of the tile: this copy's columns, zeros for the other copies'
#pragma unroll
        for (int x = 0; x < NC / 2; x += 16) tmem_st16(tS + col0 / 2 + x, p + x);
        if constexpr (R > 1) {
#pragma unroll
          for (int c = 0; c < 64; c += 16)
            if (c < col0 / 2 || c >= col0 / 2 + NC / 2) tmem_st16(tS + c, zero);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&sm.p_full[i]);
        float tmp = mc; mc = mx_; mx_ = tmp;
        tmp = lc; lc = lx; lx = tmp;
        tmp = lrc; lrc = lrx; lrx = tmp;
      }
      if (!ok) break;
      // after n swaps, stream 0's state is (mc, ...) when n is even, (mx_, ...) when odd
      const bool odd = s.n & 1;
      const float m0 = odd ? mx_ : mc, l0 = odd ? lx : lc, lr0 = odd ? lrx : lrc;
      const float m1 = odd ? mc : mx_, l1 = odd ? lc : lx, lr1 = odd ? lrc : lrx;
      const bool has1 = s.n > 1;
      ok = __all_sync(kFull, mbar_wait(&sm.o_done[0], ocnt0 & 1, wc));
      if (!ok) break;
      ++ocnt0;
      if (has1) {
        ok = __all_sync(kFull, mbar_wait(&sm.o_done[1], ocnt1 & 1, wc));
        if (!ok) break;
        ++ocnt1;
      }
      tc_fence_after();
      const float mm = fmaxf(m0, m1);
      float a0 = 0.f, a1 = 0.f;
      if (mm != -INFINITY) {
        a0 = ex2_approx(m0 - mm);
        a1 = ex2_approx(m1 - mm);
      }
      const float lsum = a0 * l0 + a1 * l1;
      const float lrsum = a0 * lr0 + a1 * lr1;
      const float inv = lrsum > 0.f ? 1.0f / lrsum : 0.f;
      const float lse_l = lsum > 0.f ? (mm + lg2_approx(lsum)) * kLn2 : -INFINITY;
      const float lse_r = lrsum > 0.f ? (mm + lg2_approx(lrsum)) * kLn2 : -INFINITY;
      const bool real = rc < M;
      const bool direct = R == 1 && s.whole;
      const int iq = rc / G;  // new position of this row
      const int b = s.p / a.H_kv;
      const int h = (s.p - b * a.H_kv) * G + (rc - iq * G);
      const int64_t slot = (static_cast<int64_t>(blockIdx.x) + s.p) * R + cp;
#pragma unroll 1
      for (int c = 0; c < D; c += 32) {
        uint32_t o0[32], o1[32];
        tmem_ld32(tO0 + c, o0);
        if (has1) tmem_ld32(tO0 + D + c, o1);
        tmem_wait_ld();
        float v[32];
#pragma unroll
        for (int x = 0; x < 32; ++x)
          v[x] = (a0 * __uint_as_float(o0[x]) + (has1 ? a1 * __uint_as_float(o1[x]) : 0.f)) * inv;
        if (real) {
          if (direct && FA_IN_BOUNDS(((static_cast<int64_t>(b) * a.N_q + iq) * a.H + h) * D + c + 32 <=
                                         static_cast<int64_t>(a.B) * a.N_q * a.H * D,
                                     status, 303)) {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<typename ElemOps<E>::T*>(a.out) +
                                                  ((static_cast<int64_t>(b) * a.N_q + iq) * a.H + h) * D + c);
#pragma unroll
            for (int x = 0; x < 4; ++x)
              dst[x] = make_uint4(ElemOps<E>::pack(v[8 * x], v[8 * x + 1]), ElemOps<E>::pack(v[8 * x + 2], v[8 * x + 3]),
                                  ElemOps<E>::pack(v[8 * x + 4], v[8 * x + 5]),
                                  ElemOps<E>::pack(v[8 * x + 6], v[8 * x + 7]));
          } else if (!direct && FA_IN_BOUNDS(slot >= 0 && slot < a.slots, status, 304)) {
            float4* dst = reinterpret_cast<float4*>(a.part_o + (slot * M + rc) * D + c);
#pragma unroll
            for (int x = 0; x < 8; ++x) dst[x] = make_float4(v[4 * x], v[4 * x + 1], v[4 * x + 2], v[4 * x + 3]);
          }
        }
      }
      if (real) {
        if (direct) {
          if (FA_IN_BOUNDS((static_cast<int64_t>(b) * a.H + h) * a.N_q + iq < static_cast<int64_t>(a.B) * a.H * a.N_q,
                           status, 305))
            a.lse[(static_cast<int64_t>(b) * a.H + h) * a.N_q + iq] = lse_l;
        } else if (FA_IN_BOUNDS(slot >= 0 && slot < a.slots, status, 306)) {
          a.part_lse[(slot * M + rc) * 2 + 0] = lse_l;
          a.part_lse[(slot * M + rc) * 2 + 1] = lse_r;
        }
      }
      tc_fence_before();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tbase, Cfg::kTmemCols);
  }
}

// Combines the partial results of the pairs whose tiles were split across CTAs or row
// copies: per row,
// LSE = log sum_s exp(lse_s) and O = sum_s exp(lr_s - LR) O_s with LR = log sum_s exp(lr_s),
// the same convex combination one CTA would have formed.  Pairs that one CTA covered were
// written by it; pairs with no key (empty cache) get O = 0, LSE = -inf.  One block of four
// warps per pair, one warp per row.
template <int D, Elem E = Elem::kBf16>
__global__ void __launch_bounds__(128) fa_decode_merge_kernel(const DecArgs a) {
  using T = typename ElemOps<E>::T;
  constexpr unsigned kFull = 0xffffffffu;
  const int p = blockIdx.x;
  const int b = p / a.H_kv;
  const int kvh = p - b * a.H_kv;
  const int G = a.H / a.H_kv;
  const int M = G * a.N_q;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const DecSeq q = dec_seq(a, b);
  if (q.T == 0) {
    for (int r = warp; r < M; r += 4) {
      const int iq = r / G, h = kvh * G + (r - iq * G);
      T* orow = static_cast<T*>(a.out) + ((static_cast<int64_t>(b) * a.N_q + iq) * a.H + h) * D;
      for (int c = lane; c < D; c += 32) orow[c] = ElemOps<E>::one(0.f);
      if (lane == 0) a.lse[(static_cast<int64_t>(b) * a.H + h) * a.N_q + iq] = -INFINITY;
    }
    return;
  }
  const int per = a.meta[1];
  const int start = a.meta[2 + b] + kvh * q.T;
  const int cf = start / per;
  const int cl = (start + q.T - 1) / per;
  if (cf == cl && a.R == 1) return;
  // partial results of this pair: slots (c + p) * R + copy for CTAs c in [cf, cl]
  const int s0 = (cf + p) * a.R;
  const int s1 = (cl + p) * a.R + a.R - 1;
  if (!FA_IN_BOUNDS(s0 >= 0 && s1 < a.slots && 2 + b < 2 + a.B, a.status, 307)) return;
  for (int r = warp; r < M; r += 4) {
    float mx_l = -INFINITY, mx_r = -INFINITY;
    for (int c = s0 + lane; c <= s1; c += 32) {
      const int64_t idx = (static_cast<int64_t>(c) * M + r) * 2;
      mx_l = fmaxf(mx_l, a.part_lse[idx]);
      mx_r = fmaxf(mx_r, a.part_lse[idx + 1]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mx_l = fmaxf(mx_l, __shfl_xor_sync(kFull, mx_l, o));
      mx_r = fmaxf(mx_r, __shfl_xor_sync(kFull, mx_r, o));
    }
    float s_l = 0.f, s_r = 0.f;
    if (mx_r != -INFINITY) {
      for (int c = s0 + lane; c <= s1; c += 32) {
        const int64_t idx = (static_cast<int64_t>(c) * M + r) * 2;
        s_l += expf(a.part_lse[idx] - mx_l);
        s_r += expf(a.part_lse[idx + 1] - mx_r);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      s_l += __shfl_xor_sync(kFull, s_l, o);
      s_r += __shfl_xor_sync(kFull, s_r, o);
    }
    const float lse_tot = mx_l == -INFINITY ? -INFINITY : mx_l + logf(s_l);
    const float lr_tot = mx_r == -INFINITY ? -INFINITY : mx_r + logf(s_r);
    float acc[D / 32];
#pragma unroll
    for (int j = 0; j < D / 32; ++j) acc[j] = 0.f;
    if (lr_tot != -INFINITY) {
      // 32 slots at a time: lane t computes the weight of slot base + t, then the warp sums
      // the slots' rows with the weights broadcast, loads independent of each other
      for (int base = s0; base <= s1; base += 32) {
        const int c = base + lane;
        float wl = 0.f;
        if (c <= s1) {
          const float lr_s = a.part_lse[(static_cast<int64_t>(c) * M + r) * 2 + 1];
          wl = lr_s == -INFINITY ? 0.f : expf(lr_s - lr_tot);
        }
        const int cnt = min(32, s1 - base + 1);
#pragma unroll 2
        for (int t = 0; t < cnt; ++t) {
          const float wgt = __shfl_sync(kFull, wl, t);
          const float* po = a.part_o + (static_cast<int64_t>(base + t) * M + r) * D;
#pragma unroll
          for (int j = 0; j < D / 32; ++j) acc[j] = fmaf(wgt, po[lane + 32 * j], acc[j]);
        }
      }
    }
    const int iq = r / G, h = kvh * G + (r - iq * G);
    T* orow = static_cast<T*>(a.out) + ((static_cast<int64_t>(b) * a.N_q + iq) * a.H + h) * D;
#pragma unroll
    for (int j = 0; j < D / 32; ++j) orow[lane + 32 * j] = ElemOps<E>::one(acc[j]);
    if (lane == 0) a.lse[(static_cast<int64_t>(b) * a.H + h) * a.N_q + iq] = lse_tot;
  }
}

}  // namespace fa
