// fattn.cu -- C ABI of libfattn (declared in include/fattn.h): argument
// validation, TMA tensor-map encoding and kernel launches.  Everything the
// operation computes runs in the kernels of fwd_kernel.cuh / bwd_kernels.cuh.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "fattn.h"

#include "bwd_kernels.cuh"
#include "fwd_kernel.cuh"

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
int make_head_map(CUtensorMap* map, const void* base, uint64_t heads, uint64_t N, int d) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) {
    t_last_cuda_error = "cuTensorMapEncodeTiled entry point not available";
    return FATTN_ERR_CUDA;
  }
  cuuint64_t dims[3] = {(cuuint64_t)d, N, heads};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, N * (cuuint64_t)d * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    char buf[96];
    snprintf(buf, sizeof(buf), "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
    t_last_cuda_error = buf;
    return FATTN_ERR_CUDA;
  }
  return FATTN_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Sequence length rounded up to whole 128-row tiles.
long long padded_n(int N) { return ((long long)N + 127) / 128 * 128; }

int check_shape(int B, int H, int N, int d) {
  if (B < 1 || H < 1 || N < 1) return FATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FATTN_ERR_UNSUPPORTED;
  // rows, and rows rounded up to whole tiles per head, are counted in int
  if ((long long)B * H * padded_n(N) >= (1ll << 31)) return FATTN_ERR_UNSUPPORTED;
  return FATTN_OK;
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
// device.  A slot goes to a launch only once the event recorded after the slot's
// previous launch has completed -- that launch's last CTA has returned the
// counters to 0 -- so no two kernels in flight share one.  A launch being
// captured into a CUDA graph, or one that finds every slot busy, schedules its
// units statically instead.
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

// Picks a free slot (pool locked by the caller); -1 if none is usable.
int sched_slot(SchedPool& pool, cudaStream_t st) {
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
  return -1;
}

template <int D, bool CAUSAL>
int launch_fwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const fattn::FwdArgs& a,
               cudaStream_t st) {
  auto kern = fattn::fattn_fwd_kernel<D, CAUSAL>;
  constexpr int smem = fattn::FwdCfg<D>::SMEM;
  if (int rc = set_smem(kern, smem)) return rc;
  int sms = 0, dev = 0;
  if (int rc = sm_count(&sms)) return rc;
  if (int rc = current_device(&dev)) return rc;
  const int ctas = a.num_units < sms ? a.num_units : sms;  // persistent: at most one CTA per SM
  fattn::FwdArgs args = a;
  args.sched = nullptr;
  if (CAUSAL) {
    // forward units: pairs of query tiles; pair p needs min(2p + 2, NT) key tiles,
    // and a head's keys and values take 4*N*d bytes
    const long long nt = a.num_q_tiles, np = (nt + 1) / 2;
    long long work = 0;
    for (long long p = 0; p < np; ++p) work += (2 * p + 2 < nt ? 2 * p + 2 : nt);
    causal_groups(a.num_units / (int)np, work, nt, 4ll * a.N * D, sms, &args.group_big, &args.num_big_groups);
  }
  SchedPool& pool = g_sched_pool[dev];
  std::unique_lock<std::mutex> lock(pool.mu, std::defer_lock);
  int slot = -1;
  if (CAUSAL && ctas > 1) {
    lock.lock();
    slot = sched_slot(pool, st);
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

template <int D, bool CAUSAL>
int launch_dkdv(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mdo,
                const CUtensorMap& mdk, const CUtensorMap& mdv, const fattn::BwdArgs& a, int BH, cudaStream_t st) {
  auto kern = fattn::fattn_bwd_dkdv_kernel<D, CAUSAL>;
  constexpr int smem = fattn::BwdCfg<D>::SMEM;
  if (int rc = set_smem(kern, smem)) return rc;
  dim3 grid((unsigned)((long long)BH * a.num_tiles));
  fattn::BwdArgs args = a;
  args.group_big = 1;
  args.num_big_groups = BH;
  if (CAUSAL) {
    // units: key tiles; tile t meets NT - t query tiles.  Per head the group
    // keeps the fp32 dQ accumulator, Q and dO in L2: 8*N*d bytes.
    int sms = 0;
    if (int rc = sm_count(&sms)) return rc;
    const long long nt = a.num_tiles;
    causal_groups(BH, nt * (nt + 1) / 2, nt, 8ll * a.N * D, sms, &args.group_big, &args.num_big_groups);
  }
  kern<<<grid, 384, smem, st>>>(mq, mk, mv, mdo, mdk, mdv, args);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "fattn_bwd_dkdv_kernel launch");
  return FATTN_OK;
}

struct WsParts {
  float* dvec;
  float* lse2;
  float* dq_acc;
};

// Workspace: D and LSE*log2(e) per query row, each head padded to whole 128-row
// tiles ([B*H][ceil(N/128)*128] fp32, so that every tile's statistics are one
// aligned 512-byte block), then the fp32 dQ accumulator [B*H*N, d].
size_t ws_bytes_needed(long long heads, int N, int d) {
  const size_t stat = align256((size_t)(heads * padded_n(N)) * sizeof(float));
  return 2 * stat + align256((size_t)heads * N * d * sizeof(float));
}

WsParts split_workspace(void* workspace, long long heads, int N) {
  char* ws = static_cast<char*>(workspace);
  const size_t stat = align256((size_t)(heads * padded_n(N)) * sizeof(float));
  WsParts p;
  p.dvec = reinterpret_cast<float*>(ws);
  p.lse2 = reinterpret_cast<float*>(ws + stat);
  p.dq_acc = reinterpret_cast<float*>(ws + 2 * stat);
  return p;
}

template <int D>
int launch_pre(const void* o, const void* dout, const float* lse, long long heads, int N, const WsParts& w,
               cudaStream_t st) {
  constexpr int rpb = 256 / (D / 8);
  const int np = (int)padded_n(N);
  const long long blocks = (heads * np + rpb - 1) / rpb;
  fattn::fattn_bwd_pre_kernel<D><<<(unsigned)blocks, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(o),
                                                                    static_cast<const __nv_bfloat16*>(dout), lse,
                                                                    w.dvec, w.lse2, w.dq_acc, heads, N, np);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "fattn_bwd_pre_kernel launch");
  return FATTN_OK;
}

template <int D>
int launch_dkdv_d(const void* q, const void* k, const void* v, const void* dout, void* dk, void* dv, int B, int H,
                  int N, int causal, float scale, const WsParts& w, cudaStream_t st) {
  const uint64_t heads = (uint64_t)B * H;
  CUtensorMap mq, mk, mv, mdo, mdk, mdv;
  if (int rc = make_head_map(&mq, q, heads, N, D)) return rc;
  if (int rc = make_head_map(&mdo, dout, heads, N, D)) return rc;
  if (int rc = make_head_map(&mk, k, heads, N, D)) return rc;
  if (int rc = make_head_map(&mv, v, heads, N, D)) return rc;
  if (int rc = make_head_map(&mdk, dk, heads, N, D)) return rc;
  if (int rc = make_head_map(&mdv, dv, heads, N, D)) return rc;
  fattn::BwdArgs a;
  a.lse2 = w.lse2;
  a.dvec = w.dvec;
  a.dq_acc = w.dq_acc;
  a.N = N;
  a.num_tiles = (N + 127) / 128;
  a.stat_stride = (int)padded_n(N);
  a.n_tail = N - (a.num_tiles - 1) * 128;
  a.scale = scale;
  a.scale_log2 = scale * kLog2e;
  const int BH = B * H;
  return causal ? launch_dkdv<D, true>(mq, mk, mv, mdo, mdk, mdv, a, BH, st)
                : launch_dkdv<D, false>(mq, mk, mv, mdo, mdk, mdv, a, BH, st);
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

int check_workspace(void* workspace, size_t bytes, int B, int H, int N, int d) {
  if (!workspace) return FATTN_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return FATTN_ERR_ALIGNMENT;
  if (bytes < ws_bytes_needed((long long)B * H, N, d)) return FATTN_ERR_INVALID_ARG;
  return FATTN_OK;
}

int check_common(int B, int H, int N, int d, float scale, int causal) {
  if (!std::isfinite(scale)) return FATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FATTN_ERR_INVALID_ARG;
  return check_shape(B, H, N, d);
}

}  // namespace

extern "C" {

int fattn_version(void) { return 0x000100; }

const char* fattn_status_string(int status) {
  switch (status) {
    case FATTN_OK: return "ok";
    case FATTN_ERR_INVALID_ARG: return "invalid argument";
    case FATTN_ERR_UNSUPPORTED: return "unsupported shape (need d in {64,128} and B*H*ceil(N/128)*128 < 2^31)";
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

int fattn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
              int causal, float scale, fattn_stream_t stream) {
  if (!q || !k || !v || !o || !lse) return FATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return FATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FATTN_ERR_INVALID_ARG;
  if (int rc = check_shape(B, H, N, d)) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return FATTN_ERR_ALIGNMENT;

  const uint64_t heads = (uint64_t)B * H;
  CUtensorMap mq, mk, mv;
  if (int rc = make_head_map(&mq, q, heads, N, d)) return rc;
  if (int rc = make_head_map(&mk, k, heads, N, d)) return rc;
  if (int rc = make_head_map(&mv, v, heads, N, d)) return rc;

  fattn::FwdArgs a;
  a.lse = lse;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.N = N;
  a.num_q_tiles = (N + 127) / 128;
  a.n_tail = N - (a.num_q_tiles - 1) * 128;
  a.num_units = B * H * ((a.num_q_tiles + 1) / 2);
  a.group_big = 1;
  a.num_big_groups = 1;
  a.sched = nullptr;
  a.scale_log2 = scale * kLog2e;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (d == 64) return causal ? launch_fwd<64, true>(mq, mk, mv, a, st) : launch_fwd<64, false>(mq, mk, mv, a, st);
  return causal ? launch_fwd<128, true>(mq, mk, mv, a, st) : launch_fwd<128, false>(mq, mk, mv, a, st);
}

size_t fattn_bwd_workspace_size(int B, int H, int N, int d) {
  if (check_shape(B, H, N, d) != FATTN_OK) return 0;
  return ws_bytes_needed((long long)B * H, N, d);
}

int fattn_bwd_preprocess(const void* o, const void* dout, const float* lse, int B, int H, int N, int d,
                         void* workspace, size_t workspace_bytes, fattn_stream_t stream) {
  if (!o || !dout || !lse || !workspace) return FATTN_ERR_INVALID_ARG;
  if (int rc = check_common(B, H, N, d, 1.f, 0)) return rc;
  if (!aligned16(o) || !aligned16(dout) || !aligned16(lse)) return FATTN_ERR_ALIGNMENT;
  if (int rc = check_workspace(workspace, workspace_bytes, B, H, N, d)) return rc;
  const long long heads = (long long)B * H;
  const WsParts w = split_workspace(workspace, heads, N);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return d == 64 ? launch_pre<64>(o, dout, lse, heads, N, w, st) : launch_pre<128>(o, dout, lse, heads, N, w, st);
}

int fattn_bwd_dkdv(const void* q, const void* k, const void* v, const void* dout, void* dk, void* dv, int B, int H,
                   int N, int d, int causal, float scale, void* workspace, size_t workspace_bytes,
                   fattn_stream_t stream) {
  if (!q || !k || !v || !dout || !dk || !dv || !workspace) return FATTN_ERR_INVALID_ARG;
  if (int rc = check_common(B, H, N, d, scale, causal)) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout) || !aligned16(dk) || !aligned16(dv))
    return FATTN_ERR_ALIGNMENT;
  if (int rc = check_workspace(workspace, workspace_bytes, B, H, N, d)) return rc;
  const WsParts w = split_workspace(workspace, (long long)B * H, N);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return d == 64 ? launch_dkdv_d<64>(q, k, v, dout, dk, dv, B, H, N, causal, scale, w, st)
                 : launch_dkdv_d<128>(q, k, v, dout, dk, dv, B, H, N, causal, scale, w, st);
}

int fattn_bwd_dq(void* dq, int B, int H, int N, int d, float scale, void* workspace, size_t workspace_bytes,
                 fattn_stream_t stream) {
  if (!dq || !workspace) return FATTN_ERR_INVALID_ARG;
  if (int rc = check_common(B, H, N, d, scale, 0)) return rc;
  if (!aligned16(dq)) return FATTN_ERR_ALIGNMENT;
  if (int rc = check_workspace(workspace, workspace_bytes, B, H, N, d)) return rc;
  const long long rows = (long long)B * H * N;
  const WsParts w = split_workspace(workspace, (long long)B * H, N);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return d == 64 ? launch_dq<64>(dq, rows, scale, w, st) : launch_dq<128>(dq, rows, scale, w, st);
}

int fattn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
              void* dq, void* dk, void* dv, int B, int H, int N, int d, int causal, float scale, void* workspace,
              size_t workspace_bytes, fattn_stream_t stream) {
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv || !workspace) return FATTN_ERR_INVALID_ARG;
  if (int rc = check_common(B, H, N, d, scale, causal)) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) || !aligned16(lse) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return FATTN_ERR_ALIGNMENT;
  if (int rc = check_workspace(workspace, workspace_bytes, B, H, N, d)) return rc;
  if (int rc = fattn_bwd_preprocess(o, dout, lse, B, H, N, d, workspace, workspace_bytes, stream)) return rc;
  if (int rc = fattn_bwd_dkdv(q, k, v, dout, dk, dv, B, H, N, d, causal, scale, workspace, workspace_bytes, stream))
    return rc;
  return fattn_bwd_dq(dq, B, H, N, d, scale, workspace, workspace_bytes, stream);
}

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
  if (int rc = check_common(B, H, N, d, scale, causal)) return rc;
  if (fattn_bwd_workspace_size(B, H, N, d) > (size_t)FATTN_NOALLOC_SCRATCH_BYTES) return FATTN_ERR_SCRATCH_TOO_SMALL;
  void* scratch = nullptr;
  if (int rc = noalloc_scratch(&scratch)) return rc;
  return fattn_bwd(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, causal, scale, scratch,
                   (size_t)FATTN_NOALLOC_SCRATCH_BYTES, stream);
}

}  // extern "C"
