// fa_bwd_kernel.cuh -- exact-attention backward for sm_100a, recomputing score tiles
// from the saved log-sum-exp instead of storing the N x N matrix ("Flash Attention
// Explained", institutepm.com, "Recompute during backward pass"; "What Is Flash
// Attention?", bestllmfor.com, "How Flash Attention works": recomputation).
//
// Gradients of L = sum(O * dO) with P = softmax(scale * Q K^T):
//   dV = P^T dO,   dP = dO V^T,   dS = P o (dP - D),   D_i = sum_x dO_ix O_ix,
//   dK = scale * dS^T Q,   dQ = scale * dS K.
// D_i equals the Jacobian row constant sum_t P_it dP_it because O_i = sum_t P_it v_t.
//
// Three kernels, one stream:
//   fa_bwd_pre  : D_i and LSE_i * log2 e (fp32, padded per head to whole 128-row blocks) and
//                 zeroing of the fp32 dQ accumulator (memory bound)
//   fa_bwd_main : one CTA per (batch, key/value head, 128-key block j), head-major; K_j and
//                 V_j stay in shared memory while, for every query head of the group that
//                 shares the key/value head, the 128-query blocks i that see block j
//                 (i >= j when causal, within the window when there is one) stream through:
//                   S^T  = K_j Q_i^T        (tcgen05, both operands in shared memory)
//                   dP^T = V_j dO_i^T
//                   P^T  = 2^(S^T * scale * log2 e - LSE_i * log2 e)   (one thread per key)
//                   dS^T = P^T o (dP^T - D_i)   (with the bf16 P^T that enters dV)
//                   dV_j += P^T dO_i        (A operand P^T read from tensor memory)
//                   dK_j += dS^T Q_i        (A operand dS^T read from shared memory)
//                   dQ_i  = dS K_j          (dS written to shared memory, 128-byte swizzle;
//                                           tensor-memory lanes are query rows)
//                 and a drain warpgroup copies each dQ_i tile out of tensor memory, frees it,
//                 stages its rows in shared memory and adds them into the fp32 accumulator
//                 with TMA reduce-adds (one bulk operation per 32 rows x 32 columns, issued
//                 by one thread, instead of a reduction instruction per element); dK_j, dV_j
//                 accumulate over the whole group in tensor memory and are written once at
//                 the end.
//   Per query block the MMA warp issues dP, then (once P is ready) dV and the next block's
//   S, then (once dS is ready) dK and dQ interleaved (two independent accumulators), so the
//   tensor core works while the key-row warpgroups compute dS and while the drain empties
//   the previous dQ tile.
//   fa_bwd_post : dQ = bf16(scale * accumulator)
//
// Tensor memory (512 columns):
//   [0,128)   S^T  (fp32).  Key-row warpgroup g (queries 64g..64g+63) reads columns
//             [64g, 64g+64) and writes its bf16 P^T into [64g, 64g+32), inside its own range.
//   [128,128+D) dP^T (fp32); once the key rows have read it, dQ_i (query rows on lanes), fp32
//   [256,256+D) dV_j accumulator,  [384,384+D) dK_j accumulator
//
// Shared memory: K_j, V_j; Q_i in a two-stage ring together with the block's LSE * log2 e
// and D runs; dO_i in one buffer (it is read only by the dP and dV products, early in the
// block, and is reloaded while the rest of the block runs); dS; two 32-row dQ staging slots.
//
// Warp roles (512 threads): warps 0-3 and 4-7 key rows for queries 0-63 and 64-127 of the
// block (P, dS; at the end dV and dK respectively), warps 8-11 dQ drain (warp 8 + w holds
// query rows 32w..32w+31), warp 12 loads (TMA tiles for Q, dO and bulk copies of the
// block's LSE * log2 e and D), warp 13 issues MMAs, warps 14-15 idle.
#pragma once

#include "fa_fwd_kernel.cuh"
#include "sm100_ptx.cuh"

namespace fa {

constexpr int kBwdThreads = 512;
constexpr uint32_t kBwdLaunchRegs = 128;  // 65536 / 512
constexpr uint32_t kBwdRegsKey = 112;     // two key-row warpgroups
constexpr uint32_t kBwdRegsDrain = 168;
constexpr uint32_t kBwdRegsOther = 104;
static_assert(128 * (2 * kBwdRegsKey + kBwdRegsDrain + kBwdRegsOther) <= kBwdThreads * kBwdLaunchRegs,
              "register split exceeds the launch allocation");
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct BwdCfg {
  static constexpr int kChunks = D / 64;
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kChunkBytes = 128 * 128;
  static constexpr uint32_t kColS = 0;
  static constexpr uint32_t kColDP = 128;
  static constexpr uint32_t kColDV = 256;
  static constexpr uint32_t kColDK = 384;
  static constexpr int kStageBytes = 32 * D * 4;  // one drain warp's 32 rows of dQ
};

template <int D>
struct __align__(1024) BwdSmem {
  uint8_t k[BwdCfg<D>::kTileBytes];
  uint8_t v[BwdCfg<D>::kTileBytes];
  uint8_t q[2][BwdCfg<D>::kTileBytes];
  uint8_t dO[BwdCfg<D>::kTileBytes];
  uint8_t ds[128 * 128 * 2];  // dS (queries x keys), MN-major A operand of dQ = dS K
  // dQ staging: two slots of 32 query rows x D fp32, each as D/32 boxes of 32 rows x 128
  // bytes in the 128-byte swizzle of the accumulator's tensor map
  uint8_t stg[2][BwdCfg<D>::kStageBytes];
  float lse2[2][128];         // LSE * log2(e) of the query block (+inf past the sequence)
  float dd[2][128];           // D of the query block
  uint64_t kv_full;
  uint64_t q_full[2];
  uint64_t q_empty[2];
  uint64_t do_full;
  uint64_t do_empty;
  uint64_t stg_free[2];
  uint64_t s_full;
  uint64_t dp_full;
  uint64_t p_ready;
  uint64_t ds_ready;
  uint64_t dq_full;
  uint64_t dq_free;
  uint64_t acc_done;
  uint64_t mma_drain;
  uint32_t tmem_base;
  int abort_flag;
};

// ---------------------------------------------------------------- pre
// For each (b, h) row n < N: D[bh, n] = sum_x dO[b,n,h,x] * O[b,n,h,x], LSE2[bh, n] =
// LSE[b,h,n] * log2(e), and the dQ accumulator row set to zero.  D and LSE2 are laid out
// [B*H, Npad] with Npad = N rounded up to 128; rows n in [N, Npad) get D = 0 and
// LSE2 = +inf, so every 128-row block is a full, 16-byte-aligned 512-byte run and its
// padded queries have P = 0.  One group of D/8 threads per row, 16-byte loads.
template <int D, Elem E = Elem::kBf16>
__global__ void __launch_bounds__(256) fa_bwd_pre_kernel(const typename ElemOps<E>::T* __restrict__ o,
                                                         const typename ElemOps<E>::T* __restrict__ dout,
                                                         const float* __restrict__ lse,
                                                         float* __restrict__ dsum, float* __restrict__ lse2,
                                                         float* __restrict__ dq_acc, int B, int H, int N,
                                                         int* status) {
  constexpr int TPR = D / 8;  // threads per row
  const int npad = (N + 127) / 128 * 128;
  const int64_t rows = static_cast<int64_t>(B) * H * npad;
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) / TPR;
  const int part = threadIdx.x % TPR;
  float acc = 0.f;
  const int64_t bh = row / npad;
  const int n = static_cast<int>(row % npad);
  const bool live = row < rows && n < N;
  if (live) {
    const int b = static_cast<int>(bh / H), h = static_cast<int>(bh % H);
    const int64_t off = ((static_cast<int64_t>(b) * N + n) * H + h) * D + part * 8;
    [[maybe_unused]] const int64_t elems = static_cast<int64_t>(B) * N * H * D;  // checking build only
    if (!FA_IN_BOUNDS(off >= 0 && off + 8 <= elems && (bh * N + n) * D + part * 8 + 8 <= elems, status, 201)) return;
    const uint4 ov = *reinterpret_cast<const uint4*>(o + off);
    const uint4 dv = *reinterpret_cast<const uint4*>(dout + off);
    const uint32_t* op = reinterpret_cast<const uint32_t*>(&ov);
    const uint32_t* dp = reinterpret_cast<const uint32_t*>(&dv);
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const float2 a = ElemOps<E>::unpack(op[x]);
      const float2 c = ElemOps<E>::unpack(dp[x]);
      acc = fmaf(a.x, c.x, acc);
      acc = fmaf(a.y, c.y, acc);
    }
    float4* z = reinterpret_cast<float4*>(dq_acc + (bh * N + n) * D + part * 8);
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int s = TPR / 2; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
  if (row < rows && part == 0 && FA_IN_BOUNDS(row >= 0 && bh < static_cast<int64_t>(B) * H, status, 202)) {
    dsum[row] = live ? acc : 0.f;
    lse2[row] = live ? lse[bh * N + n] * 1.4426950408889634f : INFINITY;
  }
}

// ---------------------------------------------------------------- post
// dQ[b,n,h,:] = (scale * acc[b,h,n,:]) in the input type, 8 elements per thread.
template <int D, Elem E = Elem::kBf16>
__global__ void __launch_bounds__(256) fa_bwd_post_kernel(const float* __restrict__ dq_acc,
                                                          typename ElemOps<E>::T* __restrict__ dq, int B, int H, int N,
                                                          float scale, int* status) {
  constexpr int TPR = D / 8;
  const int64_t rows = static_cast<int64_t>(B) * H * N;
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) / TPR;
  const int part = threadIdx.x % TPR;
  if (row >= rows) return;
  const int64_t bh = row / N;
  const int n = static_cast<int>(row % N);
  const int b = static_cast<int>(bh / H), h = static_cast<int>(bh % H);
  if (!FA_IN_BOUNDS(row * D + part * 8 + 8 <= rows * D &&
                        ((static_cast<int64_t>(b) * N + n) * H + h) * D + part * 8 + 8 <= rows * D,
                    status, 221))
    return;
  const float4* a = reinterpret_cast<const float4*>(dq_acc + row * D + part * 8);
  const float4 a0 = a[0], a1 = a[1];
  uint4 r;
  r.x = ElemOps<E>::pack(a0.x * scale, a0.y * scale);
  r.y = ElemOps<E>::pack(a0.z * scale, a0.w * scale);
  r.z = ElemOps<E>::pack(a1.x * scale, a1.y * scale);
  r.w = ElemOps<E>::pack(a1.z * scale, a1.w * scale);
  *reinterpret_cast<uint4*>(dq + ((static_cast<int64_t>(b) * N + n) * H + h) * D + part * 8) = r;
}

// P^T for 32 queries of one key row: p = 2^(s * sl - lse2), zero where masked
// (MASKED: key beyond the sequence, query index below qlim on the diagonal block, or above
// qhi past the end of a sliding window);
// returns the 16 bf16 pairs.  One branch per chunk instead of one per element keeps the
// unrolled loop a single basic block the compiler can interleave.
template <bool MASKED, Elem E = Elem::kBf16>
__device__ __forceinline__ void bwd_p_chunk(const uint32_t (&sv)[32], const float* lse2, float2 sl2, int q0,
                                            bool key_ok, int qlim, int qhi, uint32_t* pk) {
  float4 l4[8];
#pragma unroll
  for (int y = 0; y < 8; ++y) l4[y] = reinterpret_cast<const float4*>(lse2)[y];
#pragma unroll
  for (int x = 0; x < 32; x += 4) {
    const float4 l = l4[x / 4];
    const float2 a =
        ffma2(make_float2(__uint_as_float(sv[x]), __uint_as_float(sv[x + 1])), sl2, make_float2(-l.x, -l.y));
    const float2 b = ffma2(make_float2(__uint_as_float(sv[x + 2]), __uint_as_float(sv[x + 3])), sl2,
                           make_float2(-l.z, -l.w));
    float p0 = ex2_approx(a.x), p1 = ex2_approx(a.y), p2 = ex2_approx(b.x), p3 = ex2_approx(b.y);
    if (MASKED) {
      const int ql = q0 + x;
      p0 = (key_ok && ql >= qlim && ql <= qhi) ? p0 : 0.f;
      p1 = (key_ok && ql + 1 >= qlim && ql + 1 <= qhi) ? p1 : 0.f;
      p2 = (key_ok && ql + 2 >= qlim && ql + 2 <= qhi) ? p2 : 0.f;
      p3 = (key_ok && ql + 3 >= qlim && ql + 3 <= qhi) ? p3 : 0.f;
    }
    pk[x / 2] = ElemOps<E>::pack(p0, p1);
    pk[x / 2 + 1] = ElemOps<E>::pack(p2, p3);
  }
}

// ---------------------------------------------------------------- main
template <int D, bool CAUSAL, Elem E = Elem::kBf16>
__global__ void __launch_bounds__(kBwdThreads, 1)
    fa_bwd_main_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                       const __grid_constant__ CUtensorMap tm_dq, const float* __restrict__ lse2g,
                       const float* __restrict__ dsum, typename ElemOps<E>::T* __restrict__ dk,
                       typename ElemOps<E>::T* __restrict__ dv,
                       int B, int H, int H_kv, int N, int window, float scale, int heads_per_group,
                       int* status) {
  using Cfg = BwdCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if ((smem_u32(smem_raw) & 1023u) != 0) {  // the layout relies on a 1 KB aligned base
    if (threadIdx.x == 0) atomicCAS(status, 0, 5);
    return;
  }
  BwdSmem<D>& sm = *reinterpret_cast<BwdSmem<D>*>(smem_raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nkb = (N + 127) / 128;
  const int group = H / H_kv;  // query heads sharing this key/value head
  // Order: (batch, key/value head) pairs in groups of heads_per_group; within a group, key
  // blocks heaviest first (with causal masking block j meets nkb - j query blocks), the
  // group's heads interleaved.  The CTAs resident at any time cover one or two groups, so
  // their dQ accumulator rows and Q/dO tiles stay in L2, and the grid ends on the lightest
  // blocks of the last group instead of starting the last head's heaviest block near the end.
  const int BHkv = B * H_kv;
  const int grp = blockIdx.x / (heads_per_group * nkb);
  const int g0 = grp * heads_per_group;
  const int gsz = BHkv - g0 < heads_per_group ? BHkv - g0 : heads_per_group;
  const int rem = blockIdx.x - grp * heads_per_group * nkb;
  const int bhkv = g0 + rem % gsz;
  const int j = rem / gsz;
  const int b = bhkv / H_kv, hkv = bhkv % H_kv;
  // query blocks that see key block j: i >= j when causal, and with a window only those
  // whose first query is within `window` of the block's last key
  const int i0 = CAUSAL ? j : 0;
  int i1 = nkb;
  if (window >= 0) {
    const int last = (j * 128 + 127 + window) / 128 + 1;
    i1 = last < nkb ? last : nkb;
  }
  const int nper = i1 - i0;     // query blocks per query head
  const int ni = group * nper;  // iterations: every query head of the group, every block

  if (threadIdx.x == 0) {
    sm.abort_flag = 0;
    mbar_init(&sm.kv_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.q_full[s], 1);
      mbar_init(&sm.q_empty[s], 1);
      mbar_init(&sm.stg_free[s], 1);
    }
    mbar_init(&sm.do_full, 1);
    mbar_init(&sm.do_empty, 1);
    mbar_init(&sm.s_full, 1);
    mbar_init(&sm.dp_full, 1);
    mbar_init(&sm.p_ready, 256);
    mbar_init(&sm.ds_ready, 256);
    mbar_init(&sm.dq_full, 1);
    mbar_init(&sm.dq_free, 128);
    mbar_init(&sm.acc_done, 1);
    mbar_init(&sm.mma_drain, 1);
    fence_mbar_init();
  }
  if (warp == 13) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = sm.tmem_base;

  // Each warpgroup's setmaxnreg sits at the top of the branch holding all of that
  // warpgroup's code, so every instruction after it is compiled within the new limit.
  if (warp >= 12) {
    regs_set<kBwdLaunchRegs, kBwdRegsOther>();
  if (warp == 12) {
    // ------------------------------------------------------------ loads
    const WaitCtx wc{&sm.abort_flag, status, 11};
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      tma_prefetch_desc(&tm_dq);
      mbar_arrive_expect_tx(&sm.kv_full, 2 * Cfg::kTileBytes);
      for (int c = 0; c < Cfg::kChunks; ++c) {
        if (FA_IN_BOUNDS(b < B && hkv < H_kv && j * 128 < N && c * 64 < D, status, 211)) {
          tma_load_4d(sm.k + c * Cfg::kChunkBytes, &tm_k, &sm.kv_full, c * 64, hkv, j * 128, b);
          tma_load_4d(sm.v + c * Cfg::kChunkBytes, &tm_v, &sm.kv_full, c * 64, hkv, j * 128, b);
        }
      }
    }
    const int npad = nkb * 128;
    int q_issued = 0, do_issued = 0;
    bool ok = true;
    // Q_i (ring stage idx & 1, freed by the block's dK product) and dO_i (one buffer, freed
    // by the previous block's dV product) are issued in this order, which is also the order
    // in which their buffers free up.
    for (int idx = 0; idx < ni; ++idx) {
      const int st = idx & 1;
      const int i = i0 + idx % nper;
      const int h = hkv * group + idx / nper;
      ok = __all_sync(0xffffffffu, mbar_wait(&sm.q_empty[st], ((idx >> 1) & 1) ^ 1, wc));
      if (!ok) break;
      const int64_t ridx = (static_cast<int64_t>(b) * H + h) * npad + i * 128;
      if (lane == 0) {
        // Q_i tile plus the block's LSE2 and D runs (512 bytes each, padded rows)
        mbar_arrive_expect_tx(&sm.q_full[st], Cfg::kTileBytes + 2 * 512);
        for (int c = 0; c < Cfg::kChunks; ++c)
          if (FA_IN_BOUNDS(h < H && i >= 0 && i * 128 < N && c * 64 < D, status, 212))
            tma_load_4d(sm.q[st] + c * Cfg::kChunkBytes, &tm_q, &sm.q_full[st], c * 64, h, i * 128, b);
        if (FA_IN_BOUNDS(ridx >= 0 && ridx + 128 <= static_cast<int64_t>(B) * H * npad, status, 213)) {
          bulk_load(sm.lse2[st], lse2g + ridx, 512, &sm.q_full[st]);
          bulk_load(sm.dd[st], dsum + ridx, 512, &sm.q_full[st]);
        }
      }
      ++q_issued;
      ok = __all_sync(0xffffffffu, mbar_wait(&sm.do_empty, (idx & 1) ^ 1, wc));
      if (!ok) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(&sm.do_full, Cfg::kTileBytes);
        for (int c = 0; c < Cfg::kChunks; ++c)
          if (FA_IN_BOUNDS(h < H && i >= 0 && i * 128 < N && c * 64 < D, status, 212))
            tma_load_4d(sm.dO + c * Cfg::kChunkBytes, &tm_do, &sm.do_full, c * 64, h, i * 128, b);
      }
      ++do_issued;
    }
    if (!ok && lane == 0) {
      // unwinding: wait (bounded) for the copies in flight
      mbar_wait_drain(&sm.kv_full, 0, status);
      for (int idx = (q_issued > 2 ? q_issued - 2 : 0); idx < q_issued; ++idx)
        mbar_wait_drain(&sm.q_full[idx & 1], (idx >> 1) & 1, status);
      if (do_issued > 0) mbar_wait_drain(&sm.do_full, (do_issued - 1) & 1, status);
    }
  } else if (warp == 13) {
    // ------------------------------------------------------------ MMA issuer
    {  // the whole warp walks the issuer's path; one elected lane issues each MMA and commit
      const WaitCtx wc{&sm.abort_flag, status, 12};
      constexpr uint32_t kT = ElemOps<E>::kMmaType;
      constexpr uint32_t idesc_sdp = idesc_kind_f16(128, 128, 0, 0, kT);  // K-major x K-major
      constexpr uint32_t idesc_acc = idesc_kind_f16(128, D, 0, 1, kT);    // K-major (TMEM or smem) A x MN-major B
      constexpr uint32_t idesc_dq = idesc_kind_f16(128, D, 1, 1, kT);     // MN-major A (dS) x MN-major B (K)
      const uint64_t dk_kmaj = sdesc_sw128(smem_u32(sm.k), 16, 1024);
      const uint64_t dv_kmaj = sdesc_sw128(smem_u32(sm.v), 16, 1024);
      const uint64_t dk_mn = sdesc_sw128(smem_u32(sm.k), Cfg::kChunkBytes, 1024);
      const uint64_t dds = sdesc_sw128(smem_u32(sm.ds), 128 * 128, 1024);  // dS^T as MN-major operand
      // the same buffer read as K-major rows (key k, queries contiguous): the A operand dS^T of dK
      const uint64_t dds_k = sdesc_sw128(smem_u32(sm.ds), 16, 1024);
      const uint32_t tS = tbase + Cfg::kColS, tDP = tbase + Cfg::kColDP;
      const uint32_t tDV = tbase + Cfg::kColDV, tDK = tbase + Cfg::kColDK;
      auto kmaj_gemm = [&](uint32_t tD, uint64_t da, uint64_t db) {  // (128 x d) . (128 x d)^T
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk / 4) * Cfg::kChunkBytes + (kk % 4) * 32) >> 4;
          umma_ss_w(tD, da + off, db + off, idesc_sdp, kk > 0);
        }
      };
      bool ok = __all_sync(0xffffffffu, mbar_wait(&sm.kv_full, 0, wc));
      ok = ok && __all_sync(0xffffffffu, mbar_wait(&sm.q_full[0], 0, wc));
      if (ok) {
        tc_fence_after();
        kmaj_gemm(tS, dk_kmaj, sdesc_sw128(smem_u32(sm.q[0]), 16, 1024));  // S^T for the first block
        umma_commit_w(&sm.s_full);
      }
      const uint64_t ddo_k = sdesc_sw128(smem_u32(sm.dO), 16, 1024);
      const uint64_t ddo_mn = sdesc_sw128(smem_u32(sm.dO), Cfg::kChunkBytes, 1024);
      for (int idx = 0; idx < ni && ok; ++idx) {
        const int st = idx & 1;
        const uint64_t dq_mn = sdesc_sw128(smem_u32(sm.q[st]), Cfg::kChunkBytes, 1024);
        if (idx > 0) {
          // dQ_{i-1} copied out of the dP columns
          ok = __all_sync(0xffffffffu, mbar_wait(&sm.dq_free, (idx - 1) & 1, wc));
          if (!ok) break;
        }
        ok = __all_sync(0xffffffffu, mbar_wait(&sm.do_full, idx & 1, wc));
        if (!ok) break;
        tc_fence_after();
        kmaj_gemm(tDP, dv_kmaj, ddo_k);  // dP^T = V dO^T
        umma_commit_w(&sm.dp_full);
        ok = __all_sync(0xffffffffu, mbar_wait(&sm.p_ready, idx & 1, wc));
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // dV += P^T dO   (K = 128 queries)
          umma_ts_w(tDV, tS + (kk >> 2) * 64 + (kk & 3) * 8, ddo_mn + ((kk * 2048) >> 4), idesc_acc,
                    (kk > 0) || (idx > 0));
        }
        umma_commit_w(&sm.do_empty);  // dO_i is no longer read once dP and dV complete
        if (idx + 1 < ni) {  // next block's S^T, into the columns P^T just left
          ok = __all_sync(0xffffffffu, mbar_wait(&sm.q_full[st ^ 1], ((idx + 1) >> 1) & 1, wc));
          if (!ok) break;
          tc_fence_after();
          kmaj_gemm(tS, dk_kmaj, sdesc_sw128(smem_u32(sm.q[st ^ 1]), 16, 1024));
          umma_commit_w(&sm.s_full);
        }
        ok = __all_sync(0xffffffffu, mbar_wait(&sm.ds_ready, idx & 1, wc));
        if (!ok) break;
        tc_fence_after();
        // dK += dS^T Q (dS^T read K-major from shared memory) and dQ = dS K (K = 128 keys, into
        // the dP columns), interleaved: two independent accumulators keep the tensor core full
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = ((kk / 4) * 16384 + (kk % 4) * 32) >> 4;
          umma_ss_w(tDK, dds_k + off, dq_mn + ((kk * 2048) >> 4), idesc_acc, (kk > 0) || (idx > 0));
          umma_ss_w(tDP, dds + ((kk * 2048) >> 4), dk_mn + ((kk * 2048) >> 4), idesc_dq, kk > 0);
        }
        umma_commit_w(&sm.q_empty[st]);
        umma_commit_w(&sm.dq_full);
      }
      umma_commit_w(&sm.acc_done);
      umma_commit_w(&sm.mma_drain);
      mbar_wait_drain(&sm.mma_drain, 0, status);
    }
    __syncwarp();
  }
  } else if (warp < 8) {
    // ------------------------------------------------------------ key rows: P^T, dS^T
    regs_set<kBwdLaunchRegs, kBwdRegsKey>();
    const int g = warp >> 2;          // query half: columns 64g .. 64g+63 of the block
    const int r = threadIdx.x & 127;  // key row within the block == TMEM lane
    const int kg = j * 128 + r;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tbase + Cfg::kColS + g * 64 + lane_off;
    const uint32_t tDP = tbase + Cfg::kColDP + g * 64 + lane_off;
    const float sl = scale * kLog2e;
    const float2 sl2 = make_float2(sl, sl);
    const WaitCtx wc{&sm.abort_flag, status, 13};
    uint8_t* ds_row = sm.ds + g * 16384 + (r >> 3) * 1024 + (r & 7) * 128;
    bool ok = true;
    for (int idx = 0; idx < ni && ok; ++idx) {
      const int st = idx & 1;
      const int i = i0 + idx % nper;
      ok = __all_sync(0xffffffffu, mbar_wait(&sm.q_full[st], (idx >> 1) & 1, wc));
      ok = ok && __all_sync(0xffffffffu, mbar_wait(&sm.s_full, idx & 1, wc));
      if (!ok) break;
      tc_fence_after();
      // valid (query q, key k): k < N, k <= q when causal, q <= k + window with a window;
      // q >= N has LSE = +inf -> P = 0
      const bool key_ok = kg < N;
      const int qbase = i * 128 + 64 * g;                            // first query of this half
      const int qlim = (CAUSAL && i == j) ? r - 64 * g : 0;          // diagonal block: query >= key
      const int qhi = window >= 0 ? kg + window - qbase : 1 << 30;   // query <= key + window
      const bool masked = __any_sync(0xffffffffu, !key_ok || qlim > 0 || qhi < 63);
      const float* lse2 = sm.lse2[st] + 64 * g;
      const float* dd = sm.dd[st] + 64 * g;
      // bf16 P^T of this key row for the warpgroup's 64 queries, packed in pairs; dS uses the
      // same rounded values that enter dV = P^T dO.  The two chunks share one copy of the
      // loop body (the kernel's code must fit the SM's instruction cache next to the other
      // roles' loops): each chunk's words land in p_hi and the previous chunk's move to p_lo,
      // so no register array is indexed by the loop counter.
      uint32_t p_lo[16], p_hi[16];
#pragma unroll
      for (int x = 0; x < 16; ++x) p_hi[x] = 0u;
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        uint32_t sv[32];
        tmem_ld32(tS + c * 32, sv);
        tmem_wait_ld();
        uint32_t pk[16];
        if (masked)
          bwd_p_chunk<true, E>(sv, lse2 + c * 32, sl2, c * 32, key_ok, qlim, qhi, pk);
        else
          bwd_p_chunk<false, E>(sv, lse2 + c * 32, sl2, c * 32, key_ok, qlim, qhi, pk);
        tmem_st16(tS + c * 16, pk);  // columns already read
#pragma unroll
        for (int x = 0; x < 16; ++x) {
          p_lo[x] = p_hi[x];
          p_hi[x] = pk[x];
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.p_ready);
      ok = __all_sync(0xffffffffu, mbar_wait(&sm.dp_full, idx & 1, wc));
      if (!ok) break;
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {  // p_lo holds this chunk's P^T words
        uint32_t dpv[32];
        tmem_ld32(tDP + c * 32, dpv);
        tmem_wait_ld();
        uint32_t dsk[16];
        float4 d4s[8];
#pragma unroll
        for (int y = 0; y < 8; ++y) d4s[y] = reinterpret_cast<const float4*>(dd + c * 32)[y];
#pragma unroll
        for (int x = 0; x < 32; x += 4) {
          const float4 d4 = d4s[x / 4];
          const uint32_t pa = p_lo[x / 2], pb = p_lo[x / 2 + 1];
          const float2 a = fmul2(ElemOps<E>::unpack(pa),
                                 fadd2(make_float2(__uint_as_float(dpv[x]), __uint_as_float(dpv[x + 1])),
                                       make_float2(-d4.x, -d4.y)));
          const float2 b = fmul2(ElemOps<E>::unpack(pb),
                                 fadd2(make_float2(__uint_as_float(dpv[x + 2]), __uint_as_float(dpv[x + 3])),
                                       make_float2(-d4.z, -d4.w)));
          dsk[x / 2] = ElemOps<E>::pack(a.x, a.y);
          dsk[x / 2 + 1] = ElemOps<E>::pack(b.x, b.y);
        }
        // dS into shared memory: row r of the 128-byte-swizzled MN-major layout; the
        // warpgroup's 64 queries are chunk g, queries 32c..32c+31 its 16-byte units 4c..4c+3
#pragma unroll
        for (int y = 0; y < 4; ++y) {
          const int u = (c * 4 + y) ^ (r & 7);
          *reinterpret_cast<uint4*>(ds_row + u * 16) =
              make_uint4(dsk[4 * y], dsk[4 * y + 1], dsk[4 * y + 2], dsk[4 * y + 3]);
        }
#pragma unroll
        for (int x = 0; x < 16; ++x) p_lo[x] = p_hi[x];
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&sm.ds_ready);
    }
    // final rows: warpgroup 0 writes dV_j, warpgroup 1 writes dK_j (x scale)
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&sm.acc_done, 0, wc));
    if (ok) {
      tc_fence_after();
      const uint32_t tAcc = tbase + (g == 0 ? Cfg::kColDV : Cfg::kColDK) + lane_off;
      const float mul = g == 0 ? 1.0f : scale;
      typename ElemOps<E>::T* dst = (g == 0 ? dv : dk) + ((static_cast<int64_t>(b) * N + kg) * H_kv + hkv) * D;
#pragma unroll 1
      for (int c = 0; c < D; c += 32) {
        uint32_t a[32];
        tmem_ld32(tAcc + c, a);
        tmem_wait_ld();
        if (kg < N && FA_IN_BOUNDS(kg >= 0 && ((static_cast<int64_t>(b) * N + kg) * H_kv + hkv) * D + c + 32 <=
                                                   static_cast<int64_t>(B) * N * H_kv * D,
                                   status, 214)) {
          uint4* pv = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
          for (int x = 0; x < 4; ++x)
            pv[x] = make_uint4(
                ElemOps<E>::pack(__uint_as_float(a[8 * x]) * mul, __uint_as_float(a[8 * x + 1]) * mul),
                ElemOps<E>::pack(__uint_as_float(a[8 * x + 2]) * mul, __uint_as_float(a[8 * x + 3]) * mul),
                ElemOps<E>::pack(__uint_as_float(a[8 * x + 4]) * mul, __uint_as_float(a[8 * x + 5]) * mul),
                ElemOps<E>::pack(__uint_as_float(a[8 * x + 6]) * mul, __uint_as_float(a[8 * x + 7]) * mul));
        }
      }
    }
    tc_fence_before();
  } else {
    // ------------------------------------------------------------ dQ drain (warps 8-11)
    // Warp 8 + w copies query rows 32w..32w+31 of dQ_i out of tensor memory, frees the
    // columns, writes the rows into its staging slot in the 128-byte swizzle of the
    // accumulator's tensor map, and one lane adds the slot into the fp32 accumulator with
    // D/32 TMA reduce-adds (rows past the sequence fall outside the map and are skipped).
    // Warps w and w + 2 share slot w & 1 and take turns: each waits until the other's
    // reduce-adds have finished reading the slot (stg_free).
    regs_set<kBwdLaunchRegs, kBwdRegsDrain>();
    const int w = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(w * 32) << 16;
    const uint32_t tQ = tbase + Cfg::kColDP + lane_off;
    const int slot = w & 1;
    uint8_t* stg = sm.stg[slot];
    uint8_t* my_row = stg + lane * 128;  // this lane's row inside each 32-row box
    const WaitCtx wc{&sm.abort_flag, status, 14};
    for (int idx = 0; idx < ni; ++idx) {
      bool ok = __all_sync(0xffffffffu, mbar_wait(&sm.dq_full, idx & 1, wc));
      if (!ok) break;
      tc_fence_after();
      uint32_t a[D];
#pragma unroll
      for (int c = 0; c < D; c += 32) tmem_ld32(tQ + c, a + c);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&sm.dq_free);  // the dP columns may be overwritten from here on
      // The slot's users alternate: warp w at block idx is user 2 idx, warp w + 2 user
      // 2 idx + 1; user k waits for the k-th arrival, i.e. for the phase of parity (k-1) & 1.
      if (w >= 2 || idx > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(&sm.stg_free[slot], w >= 2 ? 0u : 1u, wc));
        if (!ok) break;
      }
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
#pragma unroll
        for (int u = 0; u < 8; ++u)  // 16-byte unit u of the row lands at unit u ^ (row & 7)
          *reinterpret_cast<uint4*>(my_row + c * 4096 + ((u ^ (lane & 7)) << 4)) =
              make_uint4(a[32 * c + 4 * u], a[32 * c + 4 * u + 1], a[32 * c + 4 * u + 2], a[32 * c + 4 * u + 3]);
      }
      fence_proxy_async_smem();  // the generic-proxy stores become visible to the TMA unit
      __syncwarp();
      if (lane == 0) {
        const int q0 = (i0 + idx % nper) * 128 + 32 * w;
        const int bh = b * H + hkv * group + idx / nper;  // query head: row block of the accumulator
#pragma unroll
        for (int c = 0; c < D / 32; ++c)
          if (FA_IN_BOUNDS(bh < B * H && q0 >= 0 && q0 < nkb * 128, status, 215))
            tma_reduce_add_3d(&tm_dq, stg + c * 4096, 32 * c, q0, bh);
        bulk_commit_group();
        bulk_wait_group_read0();
        mbar_arrive(&sm.stg_free[slot]);
      }
      __syncwarp();
    }
    if (lane == 0) bulk_wait_group0();  // every reduce-add has landed before the CTA exits
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 13) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

}  // namespace fa
