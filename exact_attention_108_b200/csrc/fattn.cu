// fattn.cu -- C ABI of libfattn (declared in include/fattn.h): argument
// validation, TMA tensor-map encoding and kernel launches.  Everything the
// operation computes runs in the kernels of fwd_kernel.cuh, bwd_kernels.cuh and
// dq_kernel.cuh.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <type_traits>

#include "fattn.h"

#include "bwd_kernels.cuh"
#include "decode_kernel.cuh"
#include "dq_kernel.cuh"
#include "fwd_kernel.cuh"

namespace fattn {
constexpr int kSiteSelfTest = 0x7f1;

// One warp waits on a barrier that expects one arrival which never comes; the
// bounded wait gives up after sm100::kWaitLimitNs and records kSiteSelfTest.
__global__ void __launch_bounds__(32) fattn_selftest_wait_kernel() {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  const uint32_t b = sm100::smem_addr(&bar);
  if (threadIdx.x == 0) {
    sm100::mbar_init(b, 1);
    abort_flag = 0;
    sm100::fence_barrier_init();
  }
  __syncwarp();
  (void)sm100::mbar_wait(b, 0, &abort_flag, kSiteSelfTest);
}
}  // namespace fattn

namespace {

thread_local std::string t_last_cuda_error;

int cuda_fail(cudaError_t e, const char* what) {
  char buf[256];
  snprintf(buf, sizeof(buf), "%s: %s", what, cudaGetErrorString(e));
  t_last_cuda_error = buf;
  return FATTN_ERR_CUDA;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 3-D view [B*H][N][d] of a contiguous bf16 [B, H, N, d] tensor, box [1][128][64]
// with 128-byte swizzle: one box is 64 columns of a 128-row tile of one head.
// Rows past N inside a head read as zero and are never written, so a ragged last
// tile needs no special copy.
// head_rows: rows allocated per head (>= N; a key/value cache may hold more rows
// than are filled), 0 = N.
int make_head_map(CUtensorMap* map, const void* base, uint64_t heads, uint64_t N, int d, uint64_t head_rows = 0) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) {
    t_last_cuda_error = "cuTensorMapEncodeTiled entry point not available";
    return FATTN_ERR_CUDA;
  }
  cuuint64_t dims[3] = {(cuuint64_t)d, N, heads};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (head_rows ? head_rows : N) * (cuuint64_t)d * 2};
  // 64-column boxes with 128-byte swizzle for d = 64, 128; 32-column boxes with
  // 64-byte swizzle for d = 32, 96 (a box never reaches past a row)
  const bool wide = d % 64 == 0;
  cuuint32_t box[3] = {wide ? 64u : 32u, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, wide ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    char buf[96];
    snprintf(buf, sizeof(buf), "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
    t_last_cuda_error = buf;
    return FATTN_ERR_CUDA;
  }
  return FATTN_OK;
}

// Calls f with the head dim as a compile-time constant (validated: 32, 64, 96 or 128).
template <class F>
int by_d(int d, F&& f) {
  switch (d) {
    case 32: return f(std::integral_constant<int, 32>{});
    case 64: return f(std::integral_constant<int, 64>{});
    case 96: return f(std::integral_constant<int, 96>{});
    default: return f(std::integral_constant<int, 128>{});
  }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Sequence length rounded up to whole 128-row tiles.
long long padded_n(int N) { return ((long long)N + 127) / 128 * 128; }

// One attention problem, as every entry point describes it: B batches of H query
// heads (N_q rows each) against H_kv key/value heads (N_k rows each), head dim d.
struct Problem {
  int B, H, H_kv, N_q, N_k, d, causal;
  float scale, dropout_p;
  unsigned long long seed;
  unsigned int offset;
  long long q_heads() const { return (long long)B * H; }
  long long kv_heads() const { return (long long)B * H_kv; }
};

Problem square(int B, int H, int N, int d, int causal, float scale) {
  return Problem{B, H, H, N, N, d, causal, scale, 0.f, 0ull, 0u};
}

int check_problem(const Problem& p) {
  if (p.B < 1 || p.H < 1 || p.H_kv < 1 || p.N_q < 1 || p.N_k < 1) return FATTN_ERR_INVALID_ARG;
  if (p.H % p.H_kv != 0) return FATTN_ERR_INVALID_ARG;
  if (!std::isfinite(p.scale)) return FATTN_ERR_INVALID_ARG;
  if (p.causal != 0 && p.causal != 1) return FATTN_ERR_INVALID_ARG;
  if (!(p.dropout_p >= 0.f && p.dropout_p < 1.f)) return FATTN_ERR_INVALID_ARG;  // NaN fails too
  if (p.d != 32 && p.d != 64 && p.d != 96 && p.d != 128 && p.d != 256) return FATTN_ERR_UNSUPPORTED;
  // d = 256: the forward only (one query tile per CTA, see run_fwd), without dropout
  if (p.d == 256 && p.dropout_p > 0.f) return FATTN_ERR_UNSUPPORTED;
  // rows, and rows rounded up to whole tiles per head, are counted in int
  if (p.q_heads() * padded_n(p.N_q) >= (1ll << 31) || p.kv_heads() * padded_n(p.N_k) >= (1ll << 31))
    return FATTN_ERR_UNSUPPORTED;
  return FATTN_OK;
}

fattn::sm100::Dropout dropout_of(const Problem& p) {
  fattn::sm100::Dropout d;
  const double t = std::floor((double)p.dropout_p * 4294967296.0);
  d.threshold = t >= 4294967295.0 ? 0xFFFFFFFFu : (uint32_t)t;
  d.scale_keep = (float)(1.0 / (1.0 - (double)p.dropout_p));
  d.seed_lo = (uint32_t)(p.seed & 0xFFFFFFFFull);
  d.seed_hi = (uint32_t)(p.seed >> 32);
  d.offset = p.offset;
  return d;
}

template <class K>
int set_smem(K kernel, int bytes) {
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
  return FATTN_OK;
}

constexpr int kMaxDevices = 256;

int current_device(int* dev) {
  cudaError_t e = cudaGetDevice(dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (*dev < 0 || *dev >= kMaxDevices) {
    t_last_cuda_error = "device ordinal out of range";
    return FATTN_ERR_CUDA;
  }
  return FATTN_OK;
}

// Streaming multiprocessors of the current device (looked up once per device).
int sm_count(int* out) {
  static std::mutex mu;
  static int counts[kMaxDevices] = {};
  int dev = 0;
  if (int rc = current_device(&dev)) return rc;
  cudaError_t e;
  std::lock_guard<std::mutex> lock(mu);
  if (!counts[dev]) {
    e = cudaDeviceGetAttribute(&counts[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
  }
  *out = counts[dev];
  return FATTN_OK;
}

// Causal kernels: the heads' scheduling groups.  The units of a group run
// longest first, so a group must hold enough work that its longest unit
// (`longest` tile steps, out of `work` per head) is no more than about 2/3 of
// what each SM gets from the group, while the group's per-head working set
// (`head_bytes`) stays well inside L2.  The heads are then split into groups whose
// sizes differ by at most one (a small last group would leave its long units
// running alone at the end).
void causal_groups(int BH, long long work, long long longest, long long head_bytes, int sms, int* big,
                   int* num_big) {
  long long g = (3ll * sms * longest + 2 * work - 1) / (2 * work);
  const long long cap = (48ll << 20) / head_bytes;
  if (g > cap) g = cap;
  if (g > BH) g = BH;
  if (g < 1) g = 1;
  const int ng = (int)(BH / g), q = BH / ng, r = BH % ng;
  *big = r ? q + 1 : q;
  *num_big = r ? r : ng;
}

// Counters for the causal forward's dynamic unit claiming, kSchedSlots pairs per
// device.  A launch may use a slot once the launch that used it before has
// finished -- its last CTA returns the counters to 0 -- so no two kernels in
// flight share one.  A slot whose event (recorded after its previous launch) has
// completed is free.  When every slot is busy, as when a host thread queues many
// calls ahead of the GPU, the launch takes the least recently handed-out slot and
// its stream first waits on that slot's event: on the same stream that wait costs
// nothing, since stream order already puts the launch after the previous one.  A
// launch being captured into a CUDA graph schedules its units statically.
constexpr int kSchedSlots = 16;
static __device__ unsigned int g_fwd_sched[kSchedSlots][2];

struct SchedPool {
  std::mutex mu;
  bool ready = false;
  unsigned int* base = nullptr;
  cudaEvent_t ev[kSchedSlots] = {};
  int next = 0;
};
SchedPool g_sched_pool[kMaxDevices];

// Picks a slot (pool locked by the caller); -1 if none is usable.  *wait is set
// when the slot may still be in use and the stream must wait on its event.
int sched_slot(SchedPool& pool, cudaStream_t st, bool* wait) {
  *wait = false;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) {
    (void)cudaGetLastError();
    return -1;
  }
  if (cs != cudaStreamCaptureStatusNone) return -1;
  if (!pool.ready) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_fwd_sched) != cudaSuccess) {
      (void)cudaGetLastError();
      return -1;
    }
    for (int i = 0; i < kSchedSlots; ++i)
      if (cudaEventCreateWithFlags(&pool.ev[i], cudaEventDisableTiming) != cudaSuccess) {
        (void)cudaGetLastError();
        for (int j = 0; j < i; ++j) cudaEventDestroy(pool.ev[j]);
        return -1;
      }
    pool.base = static_cast<unsigned int*>(p);
    pool.ready = true;
  }
  for (int i = 0; i < kSchedSlots; ++i) {
    const int s = (pool.next + i) % kSchedSlots;
    const cudaError_t q = cudaEventQuery(pool.ev[s]);
    if (q == cudaSuccess) {
      pool.next = (s + 1) % kSchedSlots;
      return s;
    }
    // a busy slot: clear the not-ready status if the runtime kept it as the last
    // error, but leave any other pending error for the launch check to report
    if (q == cudaErrorNotReady && cudaPeekAtLastError() == cudaErrorNotReady) (void)cudaGetLastError();
  }
  const int s = pool.next;
  pool.next = (s + 1) % kSchedSlots;
  *wait = true;
  return s;
}

template <int D, bool CAUSAL, bool DROP>
int launch_fwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const fattn::FwdArgs& a,
               cudaStream_t st) {
  auto kern = fattn::fattn_fwd_kernel<D, CAUSAL, DROP>;
  constexpr int smem = fattn::FwdCfg<D>::SMEM;
  if (int rc = set_smem(kern, smem)) return rc;
  int sms = 0, dev = 0;
  if (int rc = sm_count(&sms)) return rc;
  if (int rc = current_device(&dev)) return rc;
  const int ctas = a.num_units < sms ? a.num_units : sms;  // persistent: at most one CTA per SM
  fattn::FwdArgs args = a;
  args.sched = nullptr;
  if (CAUSAL) {
    // forward units: pairs of query tiles, each costing the key tiles of its second
    // tile; a head's keys and values take 4*N_k*d bytes
    const int nt = a.num_q_tiles, np = (nt + 1) / 2;
    long long work = 0;
    for (int p = 0; p < np; ++p)
      work += fattn::fwd_kv_tiles(2 * p + 1 < nt ? 2 * p + 1 : nt - 1, a.num_kv_tiles, a.causal_off, true);
    const long long longest = fattn::fwd_kv_tiles(nt - 1, a.num_kv_tiles, a.causal_off, true);
    causal_groups(a.num_units / np, work, longest, 4ll * a.num_kv_tiles * 128 * D, sms, &args.group_big,
                  &args.num_big_groups);
  }
  SchedPool& pool = g_sched_pool[dev];
  std::unique_lock<std::mutex> lock(pool.mu, std::defer_lock);
  int slot = -1;
  if (CAUSAL && ctas > 1) {
    lock.lock();
    bool wait = false;
    slot = sched_slot(pool, st, &wait);
    if (slot >= 0 && wait) {
      const cudaError_t we = cudaStreamWaitEvent(st, pool.ev[slot], 0);
      if (we != cudaSuccess) return cuda_fail(we, "cudaStreamWaitEvent");
    }
    if (slot >= 0) args.sched = pool.base + 2 * slot;
  }
  kern<<<dim3((unsigned)ctas), 384, smem, st>>>(mq, mk, mv, args);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "fattn_fwd_kernel launch");
  if (slot >= 0) {
    e = cudaEventRecord(pool.ev[slot], st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  }
  return FATTN_OK;
}

constexpr float kLog2e = 1.4426950408889634f;

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

template <int D>
int fwd_dispatch(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const fattn::FwdArgs& a,
                 bool causal, bool drop, cudaStream_t st) {
  if (causal)
    return drop ? launch_fwd<D, true, true>(mq, mk, mv, a, st) : launch_fwd<D, true, false>(mq, mk, mv, a, st);
  return drop ? launch_fwd<D, false, true>(mq, mk, mv, a, st) : launch_fwd<D, false, false>(mq, mk, mv, a, st);
}

int decode_impl(const fattn_decode_params* x, cudaStream_t st);

// The forward of a validated problem (pointers checked by the caller).
int run_fwd(const Problem& p, const void* q, const void* k, const void* v, void* o, float* lse, cudaStream_t st) {
  if (p.d == 256) {
    // Two query tiles with their 256-column O accumulators do not fit in the 512 TMEM
    // columns, so d = 256 runs the one-tile-per-CTA kernel of the decoding path with
    // a single key split (it writes O and LSE itself and needs no workspace).
    fattn_decode_params x{q, k, v, o, lse, p.B, p.H, p.H_kv, p.N_q, p.N_k, p.N_k, p.d, p.causal, p.scale, 1,
                          nullptr, 0};
    return decode_impl(&x, st);
  }
  CUtensorMap mq, mk, mv;
  if (int rc = make_head_map(&mq, q, p.q_heads(), p.N_q, p.d)) return rc;
  if (int rc = make_head_map(&mk, k, p.kv_heads(), p.N_k, p.d)) return rc;
  if (int rc = make_head_map(&mv, v, p.kv_heads(), p.N_k, p.d)) return rc;
  fattn::FwdArgs a;
  a.lse = lse;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.N_q = p.N_q;
  a.num_q_tiles = (p.N_q + 127) / 128;
  a.num_kv_tiles = (p.N_k + 127) / 128;
  a.kv_tail = p.N_k - (a.num_kv_tiles - 1) * 128;
  a.causal_off = p.N_k - p.N_q;
  a.G = p.H / p.H_kv;
  a.num_units = (int)(p.q_heads() * ((a.num_q_tiles + 1) / 2));
  a.group_big = 1;
  a.num_big_groups = 1;
  a.sched = nullptr;
  a.scale_log2 = p.scale * kLog2e;
  a.drop = dropout_of(p);
  const bool drop = p.dropout_p > 0.f;
  return by_d(p.d, [&](auto D) { return fwd_dispatch<D.value>(mq, mk, mv, a, p.causal, drop, st); });
}

// ------------------------------------------------------------------ backward
template <int D, bool CAUSAL, bool DROP, bool WITH_DQ>
int launch_dkdv(const CUtensorMap* m, const fattn::BwdArgs& a, long long kv_heads, cudaStream_t st) {
  auto kern = fattn::fattn_bwd_dkdv_kernel<D, CAUSAL, DROP, WITH_DQ>;
  constexpr int smem = fattn::BwdCfg<D>::SMEM;
  if (int rc = set_smem(kern, smem)) return rc;
  dim3 grid((unsigned)(kv_heads * a.num_kv_tiles));
  fattn::BwdArgs args = a;
  args.group_big = 1;
  args.num_big_groups = (int)kv_heads;
  if (CAUSAL) {
    // units: key tiles; tile t meets G * (NT - first query tile) query tiles.  Per
    // key/value head the group keeps the fp32 dQ accumulator, Q and dO of its query
    // heads in L2: about 8*N_q*d*G bytes.
    int sms = 0;
    if (int rc = sm_count(&sms)) return rc;
    long long work = 0, longest = 0;
    for (int t = 0; t < a.num_kv_tiles; ++t) {
      const long long n = (long long)a.G * (a.num_q_tiles - fattn::bwd_first_q_tile(t, a.causal_off, true));
      work += n;
      longest = n > longest ? n : longest;
    }
    causal_groups((int)kv_heads, work, longest, 8ll * a.num_q_tiles * 128 * D * a.G, sms, &args.group_big,
                  &args.num_big_groups);
  }
  kern<<<grid, 384, smem, st>>>(m[0], m[1], m[2], m[3], m[4], m[5], args);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "fattn_bwd_dkdv_kernel launch");
  return FATTN_OK;
}

template <int D, bool CAUSAL, bool DROP>
int launch_dq_pass(const CUtensorMap* m, const fattn::DqArgs& a, long long q_heads, cudaStream_t st) {
  auto kern = fattn::fattn_bwd_dq_pass_kernel<D, CAUSAL, DROP>;
  constexpr int smem = fattn::DqCfg<D>::SMEM;
  if (int rc = set_smem(kern, smem)) return rc;
  dim3 grid((unsigned)(q_heads * a.num_q_tiles));
  fattn::DqArgs args = a;
  args.group_big = 1;
  args.num_big_groups = (int)q_heads;
  if (CAUSAL) {
    // units: query tiles; tile t meets fwd_kv_tiles(t) key tiles.  Per query head
    // the group keeps its keys and values in L2: 4*N_k*d bytes.
    int sms = 0;
    if (int rc = sm_count(&sms)) return rc;
    long long work = 0;
    for (int t = 0; t < a.num_q_tiles; ++t) work += fattn::fwd_kv_tiles(t, a.num_kv_tiles, a.causal_off, true);
    const long long longest = fattn::fwd_kv_tiles(a.num_q_tiles - 1, a.num_kv_tiles, a.causal_off, true);
    causal_groups((int)q_heads, work, longest, 4ll * a.num_kv_tiles * 128 * D, sms, &args.group_big,
                  &args.num_big_groups);
  }
  kern<<<grid, 384, smem, st>>>(m[0], m[1], m[2], m[3], args);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "fattn_bwd_dq_pass_kernel launch");
  return FATTN_OK;
}

struct WsParts {
  float* dvec;
  float* lse2;
  float* dq_acc;  // null for the deterministic backward, which needs no accumulator
};

// Workspace: D and LSE*log2(e) per query row, each head padded to whole 128-row
// tiles ([B*H][ceil(N_q/128)*128] fp32, so that every tile's statistics are one
// aligned 512-byte block), then (default backward only) the fp32 dQ accumulator
// [B*H*N_q, d].
size_t ws_bytes_needed(const Problem& p, bool deterministic) {
  const size_t stat = align256((size_t)(p.q_heads() * padded_n(p.N_q)) * sizeof(float));
  return 2 * stat + (deterministic ? 0 : align256((size_t)p.q_heads() * p.N_q * p.d * sizeof(float)));
}

WsParts split_workspace(void* workspace, const Problem& p, bool deterministic) {
  char* ws = static_cast<char*>(workspace);
  const size_t stat = align256((size_t)(p.q_heads() * padded_n(p.N_q)) * sizeof(float));
  WsParts w;
  w.dvec = reinterpret_cast<float*>(ws);
  w.lse2 = reinterpret_cast<float*>(ws + stat);
  w.dq_acc = deterministic ? nullptr : reinterpret_cast<float*>(ws + 2 * stat);
  return w;
}

template <int D>
int launch_pre(const void* o, const void* dout, const float* lse, const Problem& p, const WsParts& w,
               cudaStream_t st) {
  constexpr int rpb = 256 / (D / 8);
  const int np = (int)padded_n(p.N_q);
  const long long blocks = (p.q_heads() * np + rpb - 1) / rpb;
  fattn::fattn_bwd_pre_kernel<D><<<(unsigned)blocks, 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dout), lse, w.dvec, w.lse2, w.dq_acc,
      p.q_heads(), p.N_q, np);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "fattn_bwd_pre_kernel launch");
  return FATTN_OK;
}

template <int D>
int dkdv_dispatch(const CUtensorMap* m, const fattn::BwdArgs& a, long long kv_heads, bool causal, bool drop,
                  bool with_dq, cudaStream_t st) {
#define FATTN_DKDV(C, P, W) launch_dkdv<D, C, P, W>(m, a, kv_heads, st)
  if (causal) {
    if (drop) return with_dq ? FATTN_DKDV(true, true, true) : FATTN_DKDV(true, true, false);
    return with_dq ? FATTN_DKDV(true, false, true) : FATTN_DKDV(true, false, false);
  }
  if (drop) return with_dq ? FATTN_DKDV(false, true, true) : FATTN_DKDV(false, true, false);
  return with_dq ? FATTN_DKDV(false, false, true) : FATTN_DKDV(false, false, false);
#undef FATTN_DKDV
}

template <int D>
int dq_pass_dispatch(const CUtensorMap* m, const fattn::DqArgs& a, long long q_heads, bool causal, bool drop,
                     cudaStream_t st) {
  if (causal)
    return drop ? launch_dq_pass<D, true, true>(m, a, q_heads, st) : launch_dq_pass<D, true, false>(m, a, q_heads, st);
  return drop ? launch_dq_pass<D, false, true>(m, a, q_heads, st) : launch_dq_pass<D, false, false>(m, a, q_heads, st);
}

// Stage 2 of a validated problem: dK, dV (and, unless deterministic, dS K added
// into the accumulator).
int run_dkdv(const Problem& p, const void* q, const void* k, const void* v, const void* dout, void* dk, void* dv,
             const WsParts& w, bool deterministic, cudaStream_t st) {
  CUtensorMap m[6];  // q, k, v, dout, dk, dv
  if (int rc = make_head_map(&m[0], q, p.q_heads(), p.N_q, p.d)) return rc;
  if (int rc = make_head_map(&m[1], k, p.kv_heads(), p.N_k, p.d)) return rc;
  if (int rc = make_head_map(&m[2], v, p.kv_heads(), p.N_k, p.d)) return rc;
  if (int rc = make_head_map(&m[3], dout, p.q_heads(), p.N_q, p.d)) return rc;
  if (int rc = make_head_map(&m[4], dk, p.kv_heads(), p.N_k, p.d)) return rc;
  if (int rc = make_head_map(&m[5], dv, p.kv_heads(), p.N_k, p.d)) return rc;
  fattn::BwdArgs a;
  a.lse2 = w.lse2;
  a.dvec = w.dvec;
  a.dq_acc = w.dq_acc;
  a.N_q = p.N_q;
  a.num_q_tiles = (p.N_q + 127) / 128;
  a.num_kv_tiles = (p.N_k + 127) / 128;
  a.stat_stride = (int)padded_n(p.N_q);
  a.q_tail = p.N_q - (a.num_q_tiles - 1) * 128;
  a.kv_tail = p.N_k - (a.num_kv_tiles - 1) * 128;
  a.causal_off = p.N_k - p.N_q;
  a.G = p.H / p.H_kv;
  a.scale = p.scale;
  a.scale_log2 = p.scale * kLog2e;
  a.drop = dropout_of(p);
  const bool drop = p.dropout_p > 0.f;
  return by_d(p.d,
              [&](auto D) { return dkdv_dispatch<D.value>(m, a, p.kv_heads(), p.causal, drop, !deterministic, st); });
}

// The deterministic stage 3: dQ by the separate pass.
int run_dq_pass(const Problem& p, const void* q, const void* k, const void* v, const void* dout, void* dq,
                const WsParts& w, cudaStream_t st) {
  CUtensorMap m[4];  // q, k, v, dout
  if (int rc = make_head_map(&m[0], q, p.q_heads(), p.N_q, p.d)) return rc;
  if (int rc = make_head_map(&m[1], k, p.kv_heads(), p.N_k, p.d)) return rc;
  if (int rc = make_head_map(&m[2], v, p.kv_heads(), p.N_k, p.d)) return rc;
  if (int rc = make_head_map(&m[3], dout, p.q_heads(), p.N_q, p.d)) return rc;
  fattn::DqArgs a;
  a.lse2 = w.lse2;
  a.dvec = w.dvec;
  a.dq = static_cast<__nv_bfloat16*>(dq);
  a.N_q = p.N_q;
  a.num_q_tiles = (p.N_q + 127) / 128;
  a.num_kv_tiles = (p.N_k + 127) / 128;
  a.stat_stride = (int)padded_n(p.N_q);
  a.kv_tail = p.N_k - (a.num_kv_tiles - 1) * 128;
  a.causal_off = p.N_k - p.N_q;
  a.G = p.H / p.H_kv;
  a.scale = p.scale;
  a.scale_log2 = p.scale * kLog2e;
  a.drop = dropout_of(p);
  const bool drop = p.dropout_p > 0.f;
  return by_d(p.d, [&](auto D) { return dq_pass_dispatch<D.value>(m, a, p.q_heads(), p.causal, drop, st); });
}

template <int D>
int launch_dq(void* dq, long long rows, float scale, const WsParts& w, cudaStream_t st) {
  const long long n8 = rows * D / 8;
  long long blocks = (n8 + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  fattn::fattn_bwd_dq_kernel<D><<<(unsigned)blocks, 256, 0, st>>>(w.dq_acc, static_cast<__nv_bfloat16*>(dq), scale, n8);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "fattn_bwd_dq_kernel launch");
  return FATTN_OK;
}

// The backward's shape check: the forward's, without d = 256 (its tiles do not fit the
// backward's shared memory and TMEM).
int check_bwd_problem(const Problem& p) {
  if (int rc = check_problem(p)) return rc;
  return p.d == 256 ? FATTN_ERR_UNSUPPORTED : FATTN_OK;
}

int check_workspace(void* workspace, size_t bytes, const Problem& p, bool deterministic) {
  if (!workspace) return FATTN_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return FATTN_ERR_ALIGNMENT;
  if (bytes < ws_bytes_needed(p, deterministic)) return FATTN_ERR_INVALID_ARG;
  return FATTN_OK;
}

// The whole backward of a validated problem with checked pointers and workspace.
int run_bwd(const Problem& p, const void* q, const void* k, const void* v, const void* o, const void* dout,
            const float* lse, void* dq, void* dk, void* dv, void* workspace, bool deterministic, cudaStream_t st) {
  const WsParts w = split_workspace(workspace, p, deterministic);
  if (int rc = by_d(p.d, [&](auto D) { return launch_pre<D.value>(o, dout, lse, p, w, st); })) return rc;
  if (int rc = run_dkdv(p, q, k, v, dout, dk, dv, w, deterministic, st)) return rc;
  if (deterministic) return run_dq_pass(p, q, k, v, dout, dq, w, st);
  const long long rows = p.q_heads() * p.N_q;
  return by_d(p.d, [&](auto D) { return launch_dq<D.value>(dq, rows, p.scale, w, st); });
}

// ------------------------------------------------------------------ decoding
struct DecodePlan {
  int rows, row_tiles, num_kv_tiles, tiles_per_split, splits;
};

DecodePlan decode_plan(const fattn_decode_params& x, int sms) {
  DecodePlan pl;
  pl.rows = (x.H / x.H_kv) * x.N_q;
  pl.row_tiles = (pl.rows + 127) / 128;
  pl.num_kv_tiles = (x.N_k + 127) / 128;
  long long want = x.num_splits;
  if (want <= 0) {
    // about four CTAs per SM in all, with at least four key tiles per split
    const long long units = (long long)x.B * x.H_kv * pl.row_tiles;
    want = (4ll * sms) / units;
    const long long most = (pl.num_kv_tiles + 3) / 4;
    if (want > most) want = most;
  }
  if (want < 1) want = 1;
  if (want > pl.num_kv_tiles) want = pl.num_kv_tiles;
  pl.tiles_per_split = (int)((pl.num_kv_tiles + want - 1) / want);
  pl.splits = (pl.num_kv_tiles + pl.tiles_per_split - 1) / pl.tiles_per_split;  // none empty
  return pl;
}

int check_decode(const fattn_decode_params& x) {
  if (x.B < 1 || x.H < 1 || x.H_kv < 1 || x.N_q < 1 || x.N_k < 1) return FATTN_ERR_INVALID_ARG;
  if (x.H % x.H_kv != 0 || x.N_k_cap < x.N_k) return FATTN_ERR_INVALID_ARG;
  if (!std::isfinite(x.scale) || (x.causal != 0 && x.causal != 1) || x.num_splits < 0) return FATTN_ERR_INVALID_ARG;
  if (x.d != 32 && x.d != 64 && x.d != 96 && x.d != 128 && x.d != 256) return FATTN_ERR_UNSUPPORTED;
  const long long rows = (long long)(x.H / x.H_kv) * x.N_q;
  if ((long long)x.B * x.H_kv * ((rows + 127) / 128 * 128) >= (1ll << 31) ||
      (long long)x.B * x.H_kv * padded_n(x.N_k_cap) >= (1ll << 31))
    return FATTN_ERR_UNSUPPORTED;
  return FATTN_OK;
}

size_t decode_ws_bytes(const fattn_decode_params& x, const DecodePlan& pl) {
  if (pl.splits == 1) return 0;
  const size_t rows_all = (size_t)pl.splits * x.B * x.H_kv * pl.rows;
  return align256(rows_all * x.d * sizeof(float)) + align256(rows_all * sizeof(float));
}

template <int D, bool CAUSAL>
int launch_decode(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const fattn::DecodeArgs& a,
                  cudaStream_t st) {
  auto kern = fattn::fattn_decode_kernel<D, CAUSAL>;
  constexpr int smem = fattn::DecodeCfg<D>::SMEM;
  if (int rc = set_smem(kern, smem)) return rc;
  const unsigned grid = (unsigned)((long long)a.splits * a.kv_heads * a.row_tiles);
  kern<<<grid, 192, smem, st>>>(mq, mk, mv, a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "fattn_decode_kernel launch");
  if (a.splits > 1) {
    const long long rows = (long long)a.kv_heads * a.rows;
    fattn::fattn_decode_merge_kernel<D><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "fattn_decode_merge_kernel launch");
  }
  return FATTN_OK;
}

Problem problem_of(const fattn_fwd_params& x) {
  return Problem{x.B, x.H, x.H_kv, x.N_q, x.N_k, x.d, x.causal, x.scale, x.dropout_p, x.seed, x.offset};
}
Problem problem_of(const fattn_bwd_params& x) {
  return Problem{x.B, x.H, x.H_kv, x.N_q, x.N_k, x.d, x.causal, x.scale, x.dropout_p, x.seed, x.offset};
}

}  // namespace

extern "C" {

int fattn_version(void) { return 0x000200; }

const char* fattn_status_string(int status) {
  switch (status) {
    case FATTN_OK: return "ok";
    case FATTN_ERR_INVALID_ARG: return "invalid argument";
    case FATTN_ERR_UNSUPPORTED:
      return "unsupported shape (need d in {32,64,96,128}, or 256 for the forward and decoding without dropout, "
             "and B*H*ceil(N_q/128)*128, B*H_kv*ceil(N_k/128)*128 < 2^31)";
    case FATTN_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case FATTN_ERR_CUDA: return "CUDA error (see fattn_last_cuda_error)";
    case FATTN_ERR_DEVICE_TIMEOUT: return "a kernel wait timed out on the device";
    case FATTN_ERR_SCRATCH_TOO_SMALL:
      return "shape needs more scratch than fattn_bwd_noalloc has (FATTN_NOALLOC_SCRATCH_BYTES)";
    default: return "unknown status";
  }
}

const char* fattn_last_cuda_error(void) { return t_last_cuda_error.c_str(); }

int fattn_device_status(int clear) {
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, fattn::g_fattn_status, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "read device status");
  if (clear) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(fattn::g_fattn_status, &zero, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "clear device status");
  }
  return v == 0 ? FATTN_OK : FATTN_ERR_DEVICE_TIMEOUT;
}

int fattn_selftest_wait_timeout(fattn_stream_t stream) {
  fattn::fattn_selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "fattn_selftest_wait_kernel launch");
  return FATTN_OK;
}

int fattn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
              int causal, float scale, fattn_stream_t stream) {
  if (!q || !k || !v || !o || !lse) return FATTN_ERR_INVALID_ARG;
  const Problem p = square(B, H, N, d, causal, scale);
  if (int rc = check_problem(p)) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return FATTN_ERR_ALIGNMENT;
  return run_fwd(p, q, k, v, o, lse, reinterpret_cast<cudaStream_t>(stream));
}

int fattn_fwd_ex(const fattn_fwd_params* x, fattn_stream_t stream) {
  if (!x || !x->q || !x->k || !x->v || !x->o || !x->lse) return FATTN_ERR_INVALID_ARG;
  const Problem p = problem_of(*x);
  if (int rc = check_problem(p)) return rc;
  if (!aligned16(x->q) || !aligned16(x->k) || !aligned16(x->v) || !aligned16(x->o) || !aligned16(x->lse))
    return FATTN_ERR_ALIGNMENT;
  return run_fwd(p, x->q, x->k, x->v, x->o, x->lse, reinterpret_cast<cudaStream_t>(stream));
}

size_t fattn_bwd_workspace_size(int B, int H, int N, int d) {
  const Problem p = square(B, H, N, d, 0, 1.f);
  if (check_bwd_problem(p) != FATTN_OK) return 0;
  return ws_bytes_needed(p, false);
}

size_t fattn_bwd_ex_workspace_size(const fattn_bwd_params* x) {
  if (!x) return 0;
  const Problem p = problem_of(*x);
  if (check_bwd_problem(p) != FATTN_OK) return 0;
  return ws_bytes_needed(p, x->deterministic != 0);
}

int fattn_bwd_preprocess(const void* o, const void* dout, const float* lse, int B, int H, int N, int d,
                         void* workspace, size_t workspace_bytes, fattn_stream_t stream) {
  if (!o || !dout || !lse || !workspace) return FATTN_ERR_INVALID_ARG;
  const Problem p = square(B, H, N, d, 0, 1.f);
  if (int rc = check_bwd_problem(p)) return rc;
  if (!aligned16(o) || !aligned16(dout) || !aligned16(lse)) return FATTN_ERR_ALIGNMENT;
  if (int rc = check_workspace(workspace, workspace_bytes, p, false)) return rc;
  const WsParts w = split_workspace(workspace, p, false);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return by_d(d, [&](auto D) { return launch_pre<D.value>(o, dout, lse, p, w, st); });
}

int fattn_bwd_dkdv(const void* q, const void* k, const void* v, const void* dout, void* dk, void* dv, int B, int H,
                   int N, int d, int causal, float scale, void* workspace, size_t workspace_bytes,
                   fattn_stream_t stream) {
  if (!q || !k || !v || !dout || !dk || !dv || !workspace) return FATTN_ERR_INVALID_ARG;
  const Problem p = square(B, H, N, d, causal, scale);
  if (int rc = check_bwd_problem(p)) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout) || !aligned16(dk) || !aligned16(dv))
    return FATTN_ERR_ALIGNMENT;
  if (int rc = check_workspace(workspace, workspace_bytes, p, false)) return rc;
  const WsParts w = split_workspace(workspace, p, false);
  return run_dkdv(p, q, k, v, dout, dk, dv, w, false, reinterpret_cast<cudaStream_t>(stream));
}

int fattn_bwd_dq(void* dq, int B, int H, int N, int d, float scale, void* workspace, size_t workspace_bytes,
                 fattn_stream_t stream) {
  if (!dq || !workspace) return FATTN_ERR_INVALID_ARG;
  const Problem p = square(B, H, N, d, 0, scale);
  if (int rc = check_bwd_problem(p)) return rc;
  if (!aligned16(dq)) return FATTN_ERR_ALIGNMENT;
  if (int rc = check_workspace(workspace, workspace_bytes, p, false)) return rc;
  const long long rows = p.q_heads() * N;
  const WsParts w = split_workspace(workspace, p, false);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return by_d(d, [&](auto D) { return launch_dq<D.value>(dq, rows, scale, w, st); });
}

int fattn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
              void* dq, void* dk, void* dv, int B, int H, int N, int d, int causal, float scale, void* workspace,
              size_t workspace_bytes, fattn_stream_t stream) {
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv || !workspace) return FATTN_ERR_INVALID_ARG;
  const Problem p = square(B, H, N, d, causal, scale);
  if (int rc = check_bwd_problem(p)) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) || !aligned16(lse) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return FATTN_ERR_ALIGNMENT;
  if (int rc = check_workspace(workspace, workspace_bytes, p, false)) return rc;
  return run_bwd(p, q, k, v, o, dout, lse, dq, dk, dv, workspace, false, reinterpret_cast<cudaStream_t>(stream));
}

int fattn_bwd_ex(const fattn_bwd_params* x, fattn_stream_t stream) {
  if (!x || !x->q || !x->k || !x->v || !x->o || !x->dout || !x->lse || !x->dq || !x->dk || !x->dv ||
      !x->workspace)
    return FATTN_ERR_INVALID_ARG;
  if (x->deterministic != 0 && x->deterministic != 1) return FATTN_ERR_INVALID_ARG;
  const Problem p = problem_of(*x);
  if (int rc = check_bwd_problem(p)) return rc;
  if (!aligned16(x->q) || !aligned16(x->k) || !aligned16(x->v) || !aligned16(x->o) || !aligned16(x->dout) ||
      !aligned16(x->lse) || !aligned16(x->dq) || !aligned16(x->dk) || !aligned16(x->dv))
    return FATTN_ERR_ALIGNMENT;
  const bool det = x->deterministic != 0;
  if (int rc = check_workspace(x->workspace, x->workspace_bytes, p, det)) return rc;
  return run_bwd(p, x->q, x->k, x->v, x->o, x->dout, x->lse, x->dq, x->dk, x->dv, x->workspace, det,
                 reinterpret_cast<cudaStream_t>(stream));
}

size_t fattn_decode_workspace_size(const fattn_decode_params* x) {
  if (!x || check_decode(*x) != FATTN_OK) return 0;
  int sms = 0;
  if (sm_count(&sms) != FATTN_OK) return 0;
  return decode_ws_bytes(*x, decode_plan(*x, sms));
}

int fattn_decode(const fattn_decode_params* x, fattn_stream_t stream) {
  if (!x || !x->q || !x->k || !x->v || !x->o || !x->lse) return FATTN_ERR_INVALID_ARG;
  if (int rc = check_decode(*x)) return rc;
  if (!aligned16(x->q) || !aligned16(x->k) || !aligned16(x->v) || !aligned16(x->o) || !aligned16(x->lse))
    return FATTN_ERR_ALIGNMENT;
  return decode_impl(x, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace {
// fattn_decode after validation (also the d = 256 forward).
int decode_impl(const fattn_decode_params* x, cudaStream_t st) {
  int sms = 0;
  if (int rc = sm_count(&sms)) return rc;
  const DecodePlan pl = decode_plan(*x, sms);
  const size_t need = decode_ws_bytes(*x, pl);
  if (need > 0) {
    if (!x->workspace || x->workspace_bytes < need) return FATTN_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(x->workspace) & 255u) return FATTN_ERR_ALIGNMENT;
  }
  const long long kv_heads = (long long)x->B * x->H_kv;
  CUtensorMap mq, mk, mv;
  // q (and o) viewed per key/value head: the G*N_q rows of its query heads are contiguous
  if (int rc = make_head_map(&mq, x->q, kv_heads, (uint64_t)pl.rows, x->d)) return rc;
  if (int rc = make_head_map(&mk, x->k, kv_heads, x->N_k, x->d, x->N_k_cap)) return rc;
  if (int rc = make_head_map(&mv, x->v, kv_heads, x->N_k, x->d, x->N_k_cap)) return rc;
  fattn::DecodeArgs a;
  const size_t rows_all = (size_t)pl.splits * kv_heads * pl.rows;
  a.o_part = need ? static_cast<float*>(x->workspace) : nullptr;
  a.lse_part = need ? reinterpret_cast<float*>(static_cast<char*>(x->workspace) +
                                               align256(rows_all * x->d * sizeof(float)))
                    : nullptr;
  a.o = static_cast<__nv_bfloat16*>(x->o);
  a.lse = x->lse;
  a.rows = pl.rows;
  a.row_tiles = pl.row_tiles;
  a.N_q = x->N_q;
  a.N_k = x->N_k;
  a.num_kv_tiles = pl.num_kv_tiles;
  a.tiles_per_split = pl.tiles_per_split;
  a.splits = pl.splits;
  a.kv_heads = (int)kv_heads;
  a.causal_off = x->N_k - x->N_q;
  a.scale_log2 = x->scale * kLog2e;
  if (x->d == 256)
    return x->causal ? launch_decode<256, true>(mq, mk, mv, a, st) : launch_decode<256, false>(mq, mk, mv, a, st);
  return by_d(x->d, [&](auto D) {
    return x->causal ? launch_decode<D.value, true>(mq, mk, mv, a, st) : launch_decode<D.value, false>(mq, mk, mv, a, st);
  });
}
}  // namespace

extern "C" {

// ---------------------------------------------------------------------------
// fattn_bwd_noalloc: the backward's scratch lives in this fixed device array
// instead of a caller-provided workspace.  In host code the array's name only
// stands for the symbol; its device address comes from cudaGetSymbolAddress,
// looked up once per device (with that device current) and cached.
static __device__ __align__(256) unsigned char g_fattn_noalloc_scratch[FATTN_NOALLOC_SCRATCH_BYTES];

namespace {
std::mutex g_noalloc_mutex;
void* g_noalloc_scratch_ptr[256] = {};

int noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 256) {
    t_last_cuda_error = "device ordinal out of range for the no-allocation scratch table";
    return FATTN_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_fattn_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(no-allocation scratch)");
    g_noalloc_scratch_ptr[dev] = p;
  }
  *out = g_noalloc_scratch_ptr[dev];
  return FATTN_OK;
}
}  // namespace

int fattn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                      void* dq, void* dk, void* dv, int B, int H, int N, int d, int causal, float scale,
                      fattn_stream_t stream) {
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv) return FATTN_ERR_INVALID_ARG;
  if (int rc = check_bwd_problem(square(B, H, N, d, causal, scale))) return rc;
  if (fattn_bwd_workspace_size(B, H, N, d) > (size_t)FATTN_NOALLOC_SCRATCH_BYTES) return FATTN_ERR_SCRATCH_TOO_SMALL;
  void* scratch = nullptr;
  if (int rc = noalloc_scratch(&scratch)) return rc;
  return fattn_bwd(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, causal, scale, scratch,
                   (size_t)FATTN_NOALLOC_SCRATCH_BYTES, stream);
}

}  // extern "C"
