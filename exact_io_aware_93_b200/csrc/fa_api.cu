// fa_api.cu -- the C ABI of include/fa.h: argument validation, TMA tensor maps,
// per-device kernel setup and launches of the sm_100a kernels.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "../../include/fa.h"
#include "fa_bwd_kernel.cuh"
#include "fa_decode_kernel.cuh"
#include "fa_fwd_kernel.cuh"
#include "tma_host.h"

// Device status word: [0] = first error code a kernel recorded, [1] = wait site.
__device__ int g_fa_status[2];

namespace {

constexpr int kMaxDevices = 64;

// Per-device set-up.  The first call on a device fills `ok`, `sm_count` and `status` under
// g_dev_mutex and only then publishes `probed` (release); later calls read `probed`
// (acquire) without the lock.  The kernel-attribute flags are set under the same mutex, so
// first calls from several host threads at once are safe.
struct DeviceInfo {
  std::atomic<bool> probed{false};
  bool ok = false;
  int sm_count = 0;
  int* status = nullptr;
  bool fwd_attr[3][2][2] = {};  // [element type][d==128][causal]
  bool bwd_attr[2][2][2] = {};
  bool dec_attr[2][2][4] = {};  // [fp16][d==128][M = 128; M = 64 with 1, 2, 4 row copies]
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mutex;

// Runs `setup` (which returns true on success) once per flag, under g_dev_mutex.
template <typename F>
bool once_per_device(bool& flag, F setup) {
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  if (!flag) {
    if (!setup()) {
      cudaGetLastError();
      return false;
    }
    flag = true;
  }
  return true;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// The warp-specialised kernels move registers between warpgroups with setmaxnreg; the
// split is computed for a launch at exactly fa::kLaunchRegs registers per thread.  The
// build script fails when ptxas reports another count; this check refuses to launch a
// library that was built some other way with a different count.
template <typename K>
bool launch_regs_ok(K kern, uint32_t expected) {
  cudaFuncAttributes a;
  if (cudaFuncGetAttributes(&a, kern) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return a.numRegs == static_cast<int>(expected);
}

fa_status current_device(DeviceInfo** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return FA_ERR_DEVICE;
  }
  DeviceInfo& di = g_dev[dev];
  if (!di.probed.load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    if (!di.probed.load(std::memory_order_relaxed)) {
      cudaDeviceProp prop;
      void* sym = nullptr;
      if (cudaGetDeviceProperties(&prop, dev) == cudaSuccess && prop.major == 10 && prop.minor == 0 &&
          cudaGetSymbolAddress(&sym, g_fa_status) == cudaSuccess && sym != nullptr) {
        di.ok = true;
        di.sm_count = prop.multiProcessorCount;
        di.status = static_cast<int*>(sym);
      }
      cudaGetLastError();
      di.probed.store(true, std::memory_order_release);
    }
  }
  if (!di.ok) return FA_ERR_DEVICE;
  *out = &di;
  return FA_OK;
}

fa_status check_problem(const fa_problem& p) {
  if (p.dtype != FA_DTYPE_BF16 && p.dtype != FA_DTYPE_F16 && p.dtype != FA_DTYPE_E4M3) return FA_ERR_UNSUPPORTED;
  if (p.dtype == FA_DTYPE_E4M3 && p.d != 128) return FA_ERR_UNSUPPORTED;
  if (p.H_kv < 1 || p.H_kv > p.H || (p.H_kv >= 1 && p.H % p.H_kv != 0)) return FA_ERR_INVALID_ARG;
  if (p.window < -1 || (p.window >= 0 && p.causal != 1)) return FA_ERR_INVALID_ARG;
  return FA_OK;
}

fa_status check_common(int B, int H, int N, int d, float scale, int causal) {
  if (B < 1 || H < 1 || N < 1) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.0f) || !isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  // every element index and every tile count must stay in range
  const long double elems = static_cast<long double>(B) * N * H * d;
  if (elems > static_cast<long double>(INT64_MAX / 4)) return FA_ERR_INVALID_ARG;
  const long long nkb = (static_cast<long long>(N) + 127) / 128;
  if (static_cast<long long>(B) * H * ((nkb + 1) / 2) > INT32_MAX) return FA_ERR_INVALID_ARG;
  return FA_OK;
}

template <int D, bool CAUSAL, fa::Elem E>
fa_status launch_fwd(DeviceInfo& di, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, void* o,
                     float* lse, int B, int H, int H_kv, int N, int window, float scale, cudaStream_t stream,
                     float out_scale = 1.0f) {
  using T = typename fa::FwdOut<E>::T;
  auto kern = fa::fa_fwd_kernel<D, CAUSAL, E>;
  const int smem = static_cast<int>(sizeof(fa::FwdSmem<D, E>)) + 1024;
  if (!once_per_device(di.fwd_attr[static_cast<int>(E)][D == 128][CAUSAL], [&] {
        return launch_regs_ok(kern, fa::kLaunchRegs) &&
               cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) == cudaSuccess;
      }))
    return FA_ERR_LAUNCH;
  const long long nkb = (static_cast<long long>(N) + 127) / 128;
  const long long tiles = static_cast<long long>(B) * H * ((nkb + 1) / 2);
  const int grid = static_cast<int>(tiles < di.sm_count ? tiles : di.sm_count);
  const float scale_log2 = scale * 1.4426950408889634f;
  kern<<<grid, fa::kFwdThreads, smem, stream>>>(mq, mk, mv, static_cast<T*>(o), lse, B, H, H_kv, N, window,
                                                 scale_log2, out_scale, di.status);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_LAUNCH;
  return FA_OK;
}

// Workspace: fp32 dQ accumulator [B, H, N, d], then fp32 D and fp32 LSE * log2(e), each
// [B*H, Npad] with Npad = N rounded up to a multiple of 128.
size_t bwd_ws_bytes(int B, int H, int N, int d) {
  const size_t bh = static_cast<size_t>(B) * H;
  const size_t npad = (static_cast<size_t>(N) + 127) / 128 * 128;
  return bh * static_cast<size_t>(N) * static_cast<size_t>(d) * 4 + 2 * bh * npad * 4;
}

template <int D, bool CAUSAL, fa::Elem E>
fa_status launch_bwd(DeviceInfo& di, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                     const CUtensorMap& mdo, const void* o, const void* dO, const float* lse, void* dq, void* dk,
                     void* dv, void* ws, int B, int H, int H_kv, int N, int window, float scale,
                     cudaStream_t stream) {
  using T = typename fa::ElemOps<E>::T;
  const int64_t rows = static_cast<int64_t>(B) * H * N;
  const int64_t prows = static_cast<int64_t>(B) * H * ((N + 127) / 128 * 128);
  float* dq_acc = static_cast<float*>(ws);
  float* dsum = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + rows * D * 4);
  float* lse2 = dsum + prows;
  const unsigned pre_blocks = static_cast<unsigned>((prows * (D / 8) + 255) / 256);
  const int64_t ew_threads = rows * (D / 8);
  const unsigned ew_blocks = static_cast<unsigned>((ew_threads + 255) / 256);
  auto kern = fa::fa_bwd_main_kernel<D, CAUSAL, E>;
  const int smem = static_cast<int>(sizeof(fa::BwdSmem<D>));
  // every check that can fail comes before the first launch: on error nothing is enqueued
  CUtensorMap mdq;  // the fp32 dQ accumulator, target of the main kernel's TMA reduce-adds
  if (!fa::make_dqacc_map(&mdq, dq_acc, static_cast<long long>(B) * H, N, D)) return FA_ERR_LAUNCH;
  if (!once_per_device(di.bwd_attr[E == fa::Elem::kF16][D == 128][CAUSAL], [&] {
        return launch_regs_ok(kern, fa::kBwdLaunchRegs) &&
               cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) == cudaSuccess;
      }))
    return FA_ERR_LAUNCH;
  fa::fa_bwd_pre_kernel<D, E><<<pre_blocks, 256, 0, stream>>>(static_cast<const T*>(o), static_cast<const T*>(dO),
                                                              lse, dsum, lse2, dq_acc, B, H, N, di.status);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_LAUNCH;
  const int nkb = (N + 127) / 128;
  // Heads interleaved per group of the grid order: as many (batch, key/value head) pairs as
  // keep their Q, dO, fp32 dQ rows and K, V within about 80 MB of L2.
  const long long head_bytes =
      static_cast<long long>(N) * D * (static_cast<long long>(H / H_kv) * (2 + 2 + 4) + 2 + 2);
  long long hpg = (80ll << 20) / (head_bytes > 0 ? head_bytes : 1);
  const long long bhkv = static_cast<long long>(B) * H_kv;
  hpg = hpg < 1 ? 1 : (hpg > bhkv ? bhkv : hpg);
  kern<<<B * H_kv * nkb, fa::kBwdThreads, smem, stream>>>(mq, mk, mv, mdo, mdq, lse2, dsum, static_cast<T*>(dk),
                                                           static_cast<T*>(dv), B, H, H_kv, N, window, scale,
                                                           static_cast<int>(hpg), di.status);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_LAUNCH;
  fa::fa_bwd_post_kernel<D, E><<<ew_blocks, 256, 0, stream>>>(dq_acc, static_cast<T*>(dq), B, H, N, scale,
                                                               di.status);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_LAUNCH;
  return FA_OK;
}

template <fa::Elem E>
fa_status dispatch_fwd(DeviceInfo& di, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, void* o,
                       float* lse, const fa_problem& p, cudaStream_t s) {
  const int w = p.window;
  if (p.d == 128)
    return p.causal ? launch_fwd<128, true, E>(di, mq, mk, mv, o, lse, p.B, p.H, p.H_kv, p.N, w, p.scale, s)
                    : launch_fwd<128, false, E>(di, mq, mk, mv, o, lse, p.B, p.H, p.H_kv, p.N, w, p.scale, s);
  return p.causal ? launch_fwd<64, true, E>(di, mq, mk, mv, o, lse, p.B, p.H, p.H_kv, p.N, w, p.scale, s)
                  : launch_fwd<64, false, E>(di, mq, mk, mv, o, lse, p.B, p.H, p.H_kv, p.N, w, p.scale, s);
}

fa_status dispatch_fwd_e4m3(DeviceInfo& di, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                           void* o, float* lse, const fa_problem& p, float out_scale, cudaStream_t s) {
  constexpr fa::Elem E = fa::Elem::kE4M3;
  const int w = p.window;
  return p.causal ? launch_fwd<128, true, E>(di, mq, mk, mv, o, lse, p.B, p.H, p.H_kv, p.N, w, p.scale, s, out_scale)
                  : launch_fwd<128, false, E>(di, mq, mk, mv, o, lse, p.B, p.H, p.H_kv, p.N, w, p.scale, s, out_scale);
}

fa::MapElem map_elem(int dtype) {
  return dtype == FA_DTYPE_F16 ? fa::MapElem::kF16 : (dtype == FA_DTYPE_E4M3 ? fa::MapElem::kE4M3 : fa::MapElem::kBf16);
}

struct BwdPtrs {
  const void* o;
  const void* dO;
  const float* lse;
  void* dq;
  void* dk;
  void* dv;
  void* ws;
};

template <fa::Elem E>
fa_status dispatch_bwd(DeviceInfo& di, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                       const CUtensorMap& mdo, const BwdPtrs& x, const fa_problem& p, cudaStream_t s) {
  const int B = p.B, H = p.H, H_kv = p.H_kv, N = p.N, w = p.window;
  if (p.d == 128)
    return p.causal ? launch_bwd<128, true, E>(di, mq, mk, mv, mdo, x.o, x.dO, x.lse, x.dq, x.dk, x.dv, x.ws, B, H,
                                               H_kv, N, w, p.scale, s)
                    : launch_bwd<128, false, E>(di, mq, mk, mv, mdo, x.o, x.dO, x.lse, x.dq, x.dk, x.dv, x.ws, B, H,
                                                H_kv, N, w, p.scale, s);
  return p.causal ? launch_bwd<64, true, E>(di, mq, mk, mv, mdo, x.o, x.dO, x.lse, x.dq, x.dk, x.dv, x.ws, B, H,
                                            H_kv, N, w, p.scale, s)
                  : launch_bwd<64, false, E>(di, mq, mk, mv, mdo, x.o, x.dO, x.lse, x.dq, x.dk, x.dv, x.ws, B, H,
                                             H_kv, N, w, p.scale, s);
}

// ---------------------------------------------------------------- decoding
fa_status check_decode(const fa_decode_problem& p) {
  if (p.B < 1 || p.H < 1 || p.H_kv < 1 || p.N_q < 1 || p.N_kv < 1) return FA_ERR_INVALID_ARG;
  if (p.H_kv > p.H || p.H % p.H_kv != 0) return FA_ERR_INVALID_ARG;
  if (!(p.scale > 0.0f) || !isfinite(p.scale)) return FA_ERR_INVALID_ARG;
  if (p.causal != 0 && p.causal != 1) return FA_ERR_INVALID_ARG;
  if (p.window < -1 || (p.window >= 0 && p.causal != 1)) return FA_ERR_INVALID_ARG;
  if (p.d != 64 && p.d != 128) return FA_ERR_UNSUPPORTED;
  if (p.dtype != FA_DTYPE_BF16 && p.dtype != FA_DTYPE_F16) return FA_ERR_UNSUPPORTED;
  if (static_cast<long long>(p.H / p.H_kv) * p.N_q > fa::kDecMaxRows) return FA_ERR_UNSUPPORTED;
  // tile counts, tile starts and element offsets stay in range
  const long long tiles = static_cast<long long>(p.B) * p.H_kv * ((static_cast<long long>(p.N_kv) + 127) / 128);
  if (tiles > (1ll << 30)) return FA_ERR_INVALID_ARG;
  if (static_cast<long double>(p.B) * p.N_kv * p.H_kv * p.d > static_cast<long double>(INT64_MAX / 4))
    return FA_ERR_INVALID_ARG;
  return FA_OK;
}

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

struct DecLayout {
  size_t meta, part_lse, part_o, total;
  size_t slots;  // partial results S = R * (grid + B * H_kv - 1)
};

// Workspace regions: schedule (total, tiles per CTA, per-sequence prefix), then the
// partial log-sum-exps [S, M, 2] and partial outputs [S, M, d] of S = R * (grid + B*H_kv - 1)
// slots (slot = (CTA index + pair index) * R + row copy is unique along the flattened
// tile list).
DecLayout dec_layout(const fa_decode_problem& p, int grid) {
  const size_t M = static_cast<size_t>(p.H / p.H_kv) * p.N_q;
  const size_t slots = (static_cast<size_t>(grid) + static_cast<size_t>(p.B) * p.H_kv - 1) *
                       static_cast<size_t>(fa::dec_copies(static_cast<int>(M)));
  DecLayout L;
  L.slots = slots;
  L.meta = 0;
  L.part_lse = round256((2 + static_cast<size_t>(p.B)) * 4);
  L.part_o = L.part_lse + round256(slots * M * 2 * 4);
  L.total = L.part_o + slots * M * static_cast<size_t>(p.d) * 4;
  return L;
}

template <int D, fa::Elem E>
fa_status launch_decode(DeviceInfo& di, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                        const fa_decode_problem& p, const int* seqlens, void* o, float* lse, void* ws,
                        cudaStream_t stream) {
  const int M = (p.H / p.H_kv) * p.N_q;
  const int R = fa::dec_copies(M);
  const bool m64 = fa::dec_mma_rows(M) == 64;
  auto kern = !m64 ? fa::fa_decode_kernel<D, E, 1, 128>
                   : (R == 4 ? fa::fa_decode_kernel<D, E, 4, 64>
                             : (R == 2 ? fa::fa_decode_kernel<D, E, 2, 64> : fa::fa_decode_kernel<D, E, 1, 64>));
  const int smem = static_cast<int>(sizeof(fa::DecSmem<D>)) + 1024;
  if (!once_per_device(di.dec_attr[E == fa::Elem::kF16][D == 128][m64 ? 1 + (R >> 1) : 0], [&] {
        return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) == cudaSuccess;
      }))
    return FA_ERR_LAUNCH;
  const int grid = di.sm_count;
  const DecLayout L = dec_layout(p, grid);
  uint8_t* w = static_cast<uint8_t*>(ws);
  fa::DecArgs a;
  a.seqlens = seqlens;
  a.out = o;
  a.lse = lse;
  a.meta = reinterpret_cast<int*>(w + L.meta);
  a.part_lse = reinterpret_cast<float*>(w + L.part_lse);
  a.part_o = reinterpret_cast<float*>(w + L.part_o);
  a.B = p.B;
  a.H = p.H;
  a.H_kv = p.H_kv;
  a.N_q = p.N_q;
  a.N_kv = p.N_kv;
  a.window = p.window;
  a.causal = p.causal;
  a.R = R;
  a.scale_log2 = p.scale * 1.4426950408889634f;
  a.slots = static_cast<long long>(L.slots);
  a.status = di.status;
  kern<<<grid, fa::kDecThreads, smem, stream>>>(mq, mk, mv, a, di.status);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_LAUNCH;
  fa::fa_decode_merge_kernel<D, E><<<p.B * p.H_kv, 128, 0, stream>>>(a);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_LAUNCH;
  return FA_OK;
}

// ---------------------------------------------------------------- wait-timeout self-test
// One warp waits on an mbarrier that nothing will ever arrive on, with the given bound,
// through the same bounded-wait path the attention kernels use.  The wait runs out, the
// status word records FA_ERR_TIMEOUT and the kernel returns normally.
__global__ void fa_wait_timeout_selftest_kernel(uint64_t timeout_ns, int* status) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    fa::mbar_init(&bar, 1);
    fa::fence_mbar_init();
  }
  __syncwarp();
  const fa::WaitCtx wc{&abort_flag, status, 99};
  fa::mbar_wait(&bar, 0, wc, timeout_ns);
}

// ---------------------------------------------------------------- bounds-check self-test
// One warp checks an index against a one-element target; lane 0's index is one past the
// end, so in the checking build its check fails, records FA_ERR_BOUNDS and skips the store.
// The array has a spare second element, so no build ever writes outside it.  Only the
// checking build launches it.
[[maybe_unused]] __global__ void fa_bounds_selftest_kernel(int* status) {
  __shared__ int target[2];
  const int idx = threadIdx.x == 0 ? 1 : 0;
  if (FA_IN_BOUNDS(idx < 1, status, 999)) target[idx] = static_cast<int>(threadIdx.x);
  __syncwarp();
  (void)target[0];
}

// ---------------------------------------------------------------- allocation-free backward
// Scratch for fa_bwd_noalloc: a fixed device array in this module, so callers that may not
// allocate device memory still get a backward pass.  It exists on every GPU that loads the
// library, for the life of the process, and every fa_bwd_noalloc call on a device uses it.
constexpr size_t kNoAllocScratchBytes = static_cast<size_t>(64) << 20;  // 64 MiB
static __device__ __align__(256) uint8_t g_fa_noalloc_scratch[kNoAllocScratchBytes];

struct NoAllocScratch {
  bool ready = false;
  void* ptr = nullptr;  // device address of g_fa_noalloc_scratch on this device
};
NoAllocScratch g_noalloc[kMaxDevices];
std::mutex g_noalloc_mutex;

// Per-device set-up, done once with the device current: in host code the array's name is
// only a stand-in, so the kernels get the address the runtime reports for this device.
fa_status noalloc_scratch(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return FA_ERR_DEVICE;
  }
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  NoAllocScratch& ns = g_noalloc[dev];
  if (!ns.ready) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_fa_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return FA_ERR_DEVICE;
    }
    ns.ptr = p;
    ns.ready = true;
  }
  *out = ns.ptr;
  return FA_OK;
}

}  // namespace

extern "C" {

int fa_abi_version(void) { return 6; }

int fa_checks_enabled(void) {
#ifdef FA_CHECKS
  return 1;
#else
  return 0;
#endif
}

const char* fa_status_string(int s) {
  switch (s) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
    case FA_ERR_ALIGNMENT: return "FA_ERR_ALIGNMENT";
    case FA_ERR_DEVICE: return "FA_ERR_DEVICE";
    case FA_ERR_LAUNCH: return "FA_ERR_LAUNCH";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT";
    case FA_ERR_WORKSPACE: return "FA_ERR_WORKSPACE";
    case FA_ERR_BOUNDS: return "FA_ERR_BOUNDS";
    default: return "FA_ERR_UNKNOWN";
  }
}

static fa_status fwd_common(const fa_problem* problem, const void* q, const void* k, const void* v, void* o,
                            float* lse, float q_descale, float k_descale, float v_descale, void* stream);

fa_status fa_fwd_ex(const fa_problem* problem, const void* q, const void* k, const void* v, void* o, float* lse,
                    void* stream) {
  return fwd_common(problem, q, k, v, o, lse, 1.0f, 1.0f, 1.0f, stream);
}

fa_status fa_fwd_e4m3_scaled(const fa_problem* problem, const void* q, const void* k, const void* v,
                             float q_descale, float k_descale, float v_descale, void* o, float* lse, void* stream) {
  if (!problem) return FA_ERR_INVALID_ARG;
  if (problem->dtype != FA_DTYPE_E4M3) return FA_ERR_INVALID_ARG;
  return fwd_common(problem, q, k, v, o, lse, q_descale, k_descale, v_descale, stream);
}

static fa_status fwd_common(const fa_problem* problem, const void* q, const void* k, const void* v, void* o,
                            float* lse, float q_descale, float k_descale, float v_descale, void* stream) {
  if (!problem || !q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  const fa_problem p = *problem;
  fa_status st = check_common(p.B, p.H, p.N, p.d, p.scale, p.causal);
  if (st != FA_OK) return st;
  st = check_problem(p);
  if (st != FA_OK) return st;
  for (const float x : {q_descale, k_descale, v_descale})
    if (!(x > 0.0f) || !isfinite(x)) return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4))
    return FA_ERR_ALIGNMENT;
  DeviceInfo* di = nullptr;
  st = current_device(&di);
  if (st != FA_OK) return st;
  CUtensorMap mq, mk, mv;
  const fa::MapElem me = map_elem(p.dtype);
  if (!fa::make_bshd_map(&mq, q, p.B, p.N, p.H, p.d, 128, me) ||
      !fa::make_bshd_map(&mk, k, p.B, p.N, p.H_kv, p.d, 128, me) ||
      !fa::make_bshd_map(&mv, v, p.B, p.N, p.H_kv, p.d, 128, me))
    return FA_ERR_LAUNCH;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (p.dtype == FA_DTYPE_E4M3) {
    // the dequantisation factors of Q and K scale the scores; V's scales the output
    fa_problem pe = p;
    pe.scale = p.scale * q_descale * k_descale;
    return dispatch_fwd_e4m3(*di, mq, mk, mv, o, lse, pe, v_descale, s);
  }
  return p.dtype == FA_DTYPE_F16 ? dispatch_fwd<fa::Elem::kF16>(*di, mq, mk, mv, o, lse, p, s)
                                 : dispatch_fwd<fa::Elem::kBf16>(*di, mq, mk, mv, o, lse, p, s);
}

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
                 float scale, int causal, void* stream) {
  const fa_problem p{B, H, H, N, d, scale, causal, -1, FA_DTYPE_BF16};
  return fa_fwd_ex(&p, q, k, v, o, lse, stream);
}

size_t fa_bwd_workspace_size(int B, int H, int N, int d) {
  // the same size limits as fa_bwd, so that the product below cannot wrap around
  if (check_common(B, H, N, d, 1.0f, 0) != FA_OK) return 0;
  return bwd_ws_bytes(B, H, N, d);
}

size_t fa_bwd_workspace_size_ex(const fa_problem* p) {
  if (!p) return 0;
  return fa_bwd_workspace_size(p->B, p->H, p->N, p->d);
}

fa_status fa_bwd_ex(const fa_problem* problem, const void* q, const void* k, const void* v, const void* o,
                    const void* dO, const float* lse, void* dq, void* dk, void* dv, void* workspace,
                    size_t workspace_bytes, void* stream) {
  if (!problem || !q || !k || !v || !o || !dO || !lse || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  const fa_problem p = *problem;
  const int B = p.B, H = p.H, H_kv = p.H_kv, N = p.N, d = p.d, causal = p.causal;
  const float scale = p.scale;
  fa_status st = check_common(B, H, N, d, scale, causal);
  if (st != FA_OK) return st;
  st = check_problem(p);
  if (st != FA_OK) return st;
  if (p.dtype == FA_DTYPE_E4M3) return FA_ERR_UNSUPPORTED;  // the e4m3 path is forward only
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(dO, 16) ||
      !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) || !aligned(lse, 4))
    return FA_ERR_ALIGNMENT;
  if (workspace == nullptr || workspace_bytes < bwd_ws_bytes(B, H, N, d)) return FA_ERR_WORKSPACE;
  if (!aligned(workspace, 16)) return FA_ERR_ALIGNMENT;
  if (static_cast<long long>(B) * H * ((static_cast<long long>(N) + 127) / 128) > INT32_MAX) return FA_ERR_INVALID_ARG;
  DeviceInfo* di = nullptr;
  st = current_device(&di);
  if (st != FA_OK) return st;
  CUtensorMap mq, mk, mv, mdo;
  const bool f16 = p.dtype == FA_DTYPE_F16;
  const fa::MapElem me = map_elem(p.dtype);
  if (!fa::make_bshd_map(&mq, q, B, N, H, d, 128, me) || !fa::make_bshd_map(&mk, k, B, N, H_kv, d, 128, me) ||
      !fa::make_bshd_map(&mv, v, B, N, H_kv, d, 128, me) || !fa::make_bshd_map(&mdo, dO, B, N, H, d, 128, me))
    return FA_ERR_LAUNCH;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const BwdPtrs ptr{o, dO, lse, dq, dk, dv, workspace};
  return f16 ? dispatch_bwd<fa::Elem::kF16>(*di, mq, mk, mv, mdo, ptr, p, s)
             : dispatch_bwd<fa::Elem::kBf16>(*di, mq, mk, mv, mdo, ptr, p, s);
}

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
                 void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes, int B, int H, int N, int d,
                 float scale, int causal, void* stream) {
  const fa_problem p{B, H, H, N, d, scale, causal, -1, FA_DTYPE_BF16};
  return fa_bwd_ex(&p, q, k, v, o, dO, lse, dq, dk, dv, workspace, workspace_bytes, stream);
}

fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dO,
                         const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d, float scale,
                         int causal, void* stream) {
  if (!q || !k || !v || !o || !dO || !lse || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  const fa_status st = check_common(B, H, N, d, scale, causal);
  if (st != FA_OK) return st;
  if (bwd_ws_bytes(B, H, N, d) > kNoAllocScratchBytes) return FA_ERR_WORKSPACE;
  void* scratch = nullptr;
  const fa_status ss = noalloc_scratch(&scratch);
  if (ss != FA_OK) return ss;
  return fa_bwd(q, k, v, o, dO, lse, dq, dk, dv, scratch, kNoAllocScratchBytes, B, H, N, d, scale, causal, stream);
}

size_t fa_decode_workspace_size(const fa_decode_problem* problem) {
  if (!problem || check_decode(*problem) != FA_OK) return 0;
  DeviceInfo* di = nullptr;
  if (current_device(&di) != FA_OK) return 0;
  return dec_layout(*problem, di->sm_count).total;
}

fa_status fa_decode(const fa_decode_problem* problem, const void* q, const void* k_cache, const void* v_cache,
                    const int* seqlens, void* o, float* lse, void* workspace, size_t workspace_bytes,
                    void* stream) {
  if (!problem || !q || !k_cache || !v_cache || !o || !lse) return FA_ERR_INVALID_ARG;
  const fa_decode_problem p = *problem;
  fa_status st = check_decode(p);
  if (st != FA_OK) return st;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(o, 16) || !aligned(lse, 4) ||
      !aligned(seqlens, 4))
    return FA_ERR_ALIGNMENT;
  DeviceInfo* di = nullptr;
  st = current_device(&di);
  if (st != FA_OK) return st;
  if (workspace == nullptr || workspace_bytes < dec_layout(p, di->sm_count).total) return FA_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return FA_ERR_ALIGNMENT;
  const int G = p.H / p.H_kv;
  CUtensorMap mq, mk, mv;
  const bool f16 = p.dtype == FA_DTYPE_F16;
  const fa::MapElem me = map_elem(p.dtype);
  if (!fa::make_decode_q_map(&mq, q, p.B, p.N_q, p.H, p.d, G, me) ||
      !fa::make_bshd_map(&mk, k_cache, p.B, p.N_kv, p.H_kv, p.d, 128, me) ||
      !fa::make_bshd_map(&mv, v_cache, p.B, p.N_kv, p.H_kv, p.d, 128, me))
    return FA_ERR_LAUNCH;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (f16)
    return p.d == 128 ? launch_decode<128, fa::Elem::kF16>(*di, mq, mk, mv, p, seqlens, o, lse, workspace, s)
                      : launch_decode<64, fa::Elem::kF16>(*di, mq, mk, mv, p, seqlens, o, lse, workspace, s);
  return p.d == 128 ? launch_decode<128, fa::Elem::kBf16>(*di, mq, mk, mv, p, seqlens, o, lse, workspace, s)
                    : launch_decode<64, fa::Elem::kBf16>(*di, mq, mk, mv, p, seqlens, o, lse, workspace, s);
}

fa_status fa_selftest_wait_timeout(unsigned int timeout_us, void* stream) {
  if (timeout_us == 0 || timeout_us > 1000000u) return FA_ERR_INVALID_ARG;
  DeviceInfo* di = nullptr;
  const fa_status st = current_device(&di);
  if (st != FA_OK) return st;
  fa_wait_timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint64_t>(timeout_us) * 1000u, di->status);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

fa_status fa_selftest_bounds(void* stream) {
#ifndef FA_CHECKS
  (void)stream;
  return FA_ERR_UNSUPPORTED;
#else
  DeviceInfo* di = nullptr;
  const fa_status st = current_device(&di);
  if (st != FA_OK) return st;
  fa_bounds_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(di->status);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
#endif
}

fa_status fa_get_status_site(void* stream, int* site) {
  if (site) *site = 0;
  DeviceInfo* di = nullptr;
  fa_status st = current_device(&di);
  if (st != FA_OK) return st;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_DEVICE;
  }
  int word[2] = {0, 0};
  const int zero[2] = {0, 0};
  if (cudaMemcpyFromSymbol(word, g_fa_status, sizeof(word)) != cudaSuccess ||
      cudaMemcpyToSymbol(g_fa_status, zero, sizeof(zero)) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_DEVICE;
  }
  if (site) *site = word[1];
  return word[0] == 0 ? FA_OK : static_cast<fa_status>(word[0]);
}

fa_status fa_get_status(void* stream) { return fa_get_status_site(stream, nullptr); }

}  // extern "C"
