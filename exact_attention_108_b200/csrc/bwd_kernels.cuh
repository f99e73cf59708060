// bwd_kernels.cuh -- exact-attention backward for sm_100a.
//
// The backward recomputes S and P tile by tile from Q, K and the saved
// log-sum-exp instead of reading a stored probability matrix (page 2 "四、反向
// 传播选择重计算而非全量保存").  Three kernels run in order on one stream:
//
//  1. fattn_bwd_pre_kernel   D_i = sum_c dO_ic O_ic, LSE2_i = LSE_i log2(e),
//                            and zero the fp32 dQ accumulator.     (HBM-bound)
//  2. fattn_bwd_dkdv_kernel  one CTA per (batch*head, 128-row key tile j);
//                            loops over the 128-row query tiles i that can see
//                            tile j and, on the tcgen05 tensor cores,
//                              S^T  = K_j Q_i^T          (TMEM)
//                              dP^T = V_j dO_i^T         (TMEM)
//                              P^T  = exp2(S^T scale log2e - LSE2_i)   (masked)
//                              dS^T = P^T o (dP^T - D_i)
//                              dV_j += P^T dO_i,  dK_j += dS^T Q_i  (TMEM accumulators)
//                              dQ_i += dS K_j  -> fp32 atomics into the accumulator
//                            (atomic global updates, page 3 "5.3 专用指令利用").
//  3. fattn_bwd_dq_kernel    dQ = bf16(scale * accumulator).
#pragma once

#include "sm100.cuh"

namespace fattn {

// ------------------------------------------------------------------ kernel 1
template <int D>
__global__ void __launch_bounds__(256) fattn_bwd_pre_kernel(const __nv_bfloat16* __restrict__ o,
                                                            const __nv_bfloat16* __restrict__ dout,
                                                            const float* __restrict__ lse, float* __restrict__ dvec,
                                                            float* __restrict__ lse2, float* __restrict__ dq_acc,
                                                            long long rows) {
  constexpr int TPR = D / 8;  // threads per row, 8 elements (16 bytes) each
  constexpr int RPB = 256 / TPR;
  const long long row = (long long)blockIdx.x * RPB + threadIdx.x / TPR;
  const int part = threadIdx.x % TPR;
  float acc = 0.f;
  if (row < rows) {
    const size_t off = (size_t)row * D + part * 8;
    const uint4 a = *reinterpret_cast<const uint4*>(o + off);
    const uint4 b = *reinterpret_cast<const uint4*>(dout + off);
    const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 fa = __bfloat1622float2(pa[i]);
      const float2 fb = __bfloat1622float2(pb[i]);
      acc = fmaf(fa.x, fb.x, acc);
      acc = fmaf(fa.y, fb.y, acc);
    }
    float4* z = reinterpret_cast<float4*>(dq_acc + off);
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int w = TPR / 2; w >= 1; w >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, w);
  if (row < rows && part == 0) {
    dvec[row] = acc;
    lse2[row] = lse[row] * 1.4426950408889634f;
  }
}

// ------------------------------------------------------------------ kernel 3
template <int D>
__global__ void __launch_bounds__(256) fattn_bwd_dq_kernel(const float* __restrict__ dq_acc,
                                                           __nv_bfloat16* __restrict__ dq, float scale,
                                                           long long n8) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n8;
       i += (long long)gridDim.x * blockDim.x) {
    const float4 a = reinterpret_cast<const float4*>(dq_acc)[2 * i];
    const float4 b = reinterpret_cast<const float4*>(dq_acc)[2 * i + 1];
    uint4 out;
    out.x = sm100::pack_bf16x2(a.x * scale, a.y * scale);
    out.y = sm100::pack_bf16x2(a.z * scale, a.w * scale);
    out.z = sm100::pack_bf16x2(b.x * scale, b.y * scale);
    out.w = sm100::pack_bf16x2(b.z * scale, b.w * scale);
    reinterpret_cast<uint4*>(dq)[i] = out;
  }
}

// ------------------------------------------------------------------ kernel 2
struct BwdArgs {
  const float* lse2;   // [B*H*N]  LSE * log2(e)
  const float* dvec;   // [B*H*N]  D
  float* dq_acc;       // [B*H*N, D] fp32
  __nv_bfloat16* dk;   // [B*H*N, D]
  __nv_bfloat16* dv;   // [B*H*N, D]
  int N;
  int num_tiles;       // N / 128
  float scale;         // for dK
  float scale_log2;    // scale * log2(e)
};

template <int D>
struct BwdCfg {
  static constexpr int KB = D / 64;
  static constexpr int TILE = 128 * D * 2;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = TILE;
  static constexpr int OFF_Q = 2 * TILE;
  static constexpr int OFF_DO = 3 * TILE;
  static constexpr int OFF_PT = 4 * TILE;                 // P^T  [128 kv][128 q] bf16, 32 KB
  static constexpr int OFF_DST = OFF_PT + 32768;          // dS^T [128 kv][128 q] bf16, 32 KB
  static constexpr int OFF_LSE = OFF_DST + 32768;         // 128 fp32
  static constexpr int OFF_DV = OFF_LSE + 512;            // 128 fp32
  static constexpr int OFF_BAR = OFF_DV + 512;
  // kv_full, qdo_full, qdo_empty, st_full, ds_full, dq_full, tm_free, done, drain
  static constexpr int NBAR = 9;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;
  static constexpr int TMEM_COLS = 512;
  static constexpr int TM_ST = 0, TM_DPT = 128, TM_DV = 256, TM_DK = 256 + D, TM_DQ = 128;
};

enum : int {
  kSiteBwdProducer = 0x201,
  kSiteBwdMmaKV = 0x202,
  kSiteBwdMmaQ = 0x203,
  kSiteBwdMmaFree = 0x204,
  kSiteBwdMmaDS = 0x205,
  kSiteBwdSoftS = 0x206,
  kSiteBwdSoftQ = 0x207,
  kSiteBwdSoftDQ = 0x208,
  kSiteBwdEpi = 0x209,
};

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(256, 1)
    fattn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                          const BwdArgs args) {
  using C = BwdCfg<D>;
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const uint32_t sK = sbase + C::OFF_K, sV = sbase + C::OFF_V, sQ = sbase + C::OFF_Q, sDO = sbase + C::OFF_DO;
  const uint32_t sPT = sbase + C::OFF_PT, sDST = sbase + C::OFF_DST;
  const uint32_t sLSE = sbase + C::OFF_LSE, sDvec = sbase + C::OFF_DV;
  const float* lse_s = reinterpret_cast<const float*>(smem + C::OFF_LSE);
  const float* dvec_s = reinterpret_cast<const float*>(smem + C::OFF_DV);
  const uint32_t bar0 = sbase + C::OFF_BAR;
  const uint32_t bar_kv_full = bar0, bar_qdo_full = bar0 + 8, bar_qdo_empty = bar0 + 16;
  const uint32_t bar_st_full = bar0 + 24, bar_ds_full = bar0 + 32, bar_dq_full = bar0 + 40;
  const uint32_t bar_tm_free = bar0 + 48, bar_done = bar0 + 56, bar_drain = bar0 + 64;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int NT = args.num_tiles;
  // The key tile varies fastest so that the CTAs resident at one time add into
  // the same head's dQ rows (which then stay in L2); causal: tile 0 sees the most
  // query tiles and is launched first.
  const int bh = (int)(blockIdx.x / (unsigned)NT);
  const int kv_tile = (int)(blockIdx.x % (unsigned)NT);
  const int head_row0 = bh * args.N;
  const int kv_row0 = head_row0 + kv_tile * 128;
  const int i_begin = CAUSAL ? kv_tile : 0;
  const int n_q = NT - i_begin;

  if (threadIdx.x == 0) {
    mbar_init(bar_kv_full, 1);
    mbar_init(bar_qdo_full, 1);
    mbar_init(bar_qdo_empty, 1);
    mbar_init(bar_st_full, 1);
    mbar_init(bar_ds_full, 128);
    mbar_init(bar_dq_full, 1);
    mbar_init(bar_tm_free, 128);
    mbar_init(bar_done, 1);
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
      prefetch_tensormap(&tm_do);
      mbar_arrive_expect_tx(bar_kv_full, 2 * C::TILE);
#pragma unroll
      for (int kb = 0; kb < C::KB; ++kb) {
        tma_load_2d(sK + kb * 16384, &tm_k, bar_kv_full, kb * 64, kv_row0);
        tma_load_2d(sV + kb * 16384, &tm_v, bar_kv_full, kb * 64, kv_row0);
      }
      int it = 0;
      for (; it < n_q; ++it) {
        if (!mbar_wait(bar_qdo_empty, (it & 1) ^ 1, abort_flag, kSiteBwdProducer)) break;
        const int q_row0 = head_row0 + (i_begin + it) * 128;
        mbar_arrive_expect_tx(bar_qdo_full, 2 * C::TILE + 1024);
#pragma unroll
        for (int kb = 0; kb < C::KB; ++kb) {
          tma_load_2d(sQ + kb * 16384, &tm_q, bar_qdo_full, kb * 64, q_row0);
          tma_load_2d(sDO + kb * 16384, &tm_do, bar_qdo_full, kb * 64, q_row0);
        }
        bulk_load(sLSE, args.lse2 + q_row0, 512, bar_qdo_full);
        bulk_load(sDvec, args.dvec + q_row0, 512, bar_qdo_full);
      }
      if (it < n_q) {  // aborted: let issued copies land
        mbar_wait_ns(bar_kv_full, 0, 100000000ull);
        if (it > 0) mbar_wait_ns(bar_qdo_full, (it - 1) & 1, 100000000ull);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_bf16_f32(128, 128, false, false);  // K/V (K-major) x Q/dO (K-major)
      constexpr uint32_t id_kv = idesc_bf16_f32(128, D, false, true);    // P^T/dS^T (K-major) x dO/Q (MN-major)
      constexpr uint32_t id_q = idesc_bf16_f32(128, D, true, true);      // dS (MN-major) x K (MN-major)
      bool ok = mbar_wait(bar_kv_full, 0, abort_flag, kSiteBwdMmaKV);
      for (int it = 0; it < n_q && ok; ++it) {
        if (!(ok = mbar_wait(bar_qdo_full, it & 1, abort_flag, kSiteBwdMmaQ))) break;
        if (!(ok = mbar_wait(bar_tm_free, (it & 1) ^ 1, abort_flag, kSiteBwdMmaFree))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_ss(tmem + C::TM_ST, sdesc_sw128(sK + koff, 16), sdesc_sw128(sQ + koff, 16), id_s, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_ss(tmem + C::TM_DPT, sdesc_sw128(sV + koff, 16), sdesc_sw128(sDO + koff, 16), id_s, kk > 0);
        }
        mma_commit(bar_st_full);
        if (!(ok = mbar_wait(bar_ds_full, it & 1, abort_flag, kSiteBwdMmaDS))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // K = 128 query rows
          const uint32_t aoff = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_ss(tmem + C::TM_DV, sdesc_sw128(sPT + aoff, 16), sdesc_sw128(sDO + kk * 2048, 16384), id_kv,
                 (it > 0 || kk > 0) ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t aoff = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_ss(tmem + C::TM_DK, sdesc_sw128(sDST + aoff, 16), sdesc_sw128(sQ + kk * 2048, 16384), id_kv,
                 (it > 0 || kk > 0) ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // K = 128 key rows
          mma_ss(tmem + C::TM_DQ, sdesc_sw128(sDST + kk * 2048, 16384), sdesc_sw128(sK + kk * 2048, 16384), id_q,
                 kk > 0 ? 1u : 0u);
        }
        mma_commit(bar_dq_full);
        mma_commit(bar_qdo_empty);
      }
      if (ok) mma_commit(bar_done);
      mma_commit(bar_drain);
      mbar_wait_ns(bar_drain, 0, 100000000ull);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------- softmax-gradient group
    const int wq = warp - 4;
    const int r = wq * 32 + lane;  // key row of the tile for S^T/dP^T; query row for dQ
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const float sl2 = args.scale_log2;
    bool ok = true;
    for (int it = 0; it < n_q; ++it) {
      const int i = i_begin + it;
      ok = mbar_wait(bar_st_full, it & 1, abort_flag, kSiteBwdSoftS);
      ok = ok && mbar_wait(bar_qdo_full, it & 1, abort_flag, kSiteBwdSoftQ);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const bool diag = CAUSAL && (i == kv_tile);
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        uint32_t sv[32], pv[32];
        tmem_ld32(tmem + C::TM_ST + lane_off + c4 * 32, sv);
        tmem_ld_wait(sv);
        tmem_ld32(tmem + C::TM_DPT + lane_off + c4 * 32, pv);
        tmem_ld_wait(pv);
        float p[32], ds[32];
#pragma unroll
        for (int t = 0; t < 32; ++t) {
          const int c = c4 * 32 + t;
          float e = ex2(fmaf(__uint_as_float(sv[t]), sl2, -lse_s[c]));
          if (diag && c < r) e = 0.f;
          p[t] = e;
          ds[t] = e * (__uint_as_float(pv[t]) - dvec_s[c]);
        }
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const int ch = c4 * 4 + q4;  // 16-byte chunk 0..15 along the 128 query columns
          const uint32_t off = (ch >> 3) * 16384 + sw128_offset(r, ch & 7);
          const int b = q4 * 8;
          st_shared_v4(sPT + off, pack_bf16x2(p[b], p[b + 1]), pack_bf16x2(p[b + 2], p[b + 3]),
                       pack_bf16x2(p[b + 4], p[b + 5]), pack_bf16x2(p[b + 6], p[b + 7]));
          st_shared_v4(sDST + off, pack_bf16x2(ds[b], ds[b + 1]), pack_bf16x2(ds[b + 2], ds[b + 3]),
                       pack_bf16x2(ds[b + 4], ds[b + 5]), pack_bf16x2(ds[b + 6], ds[b + 7]));
        }
      }
      fence_async_shared();
      tc_fence_before();
      mbar_arrive(bar_ds_full);
      ok = mbar_wait(bar_dq_full, it & 1, abort_flag, kSiteBwdSoftDQ);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      // dQ_i partial (TMEM lane = query row r of tile i) -> fp32 atomics.
      float* dst = args.dq_acc + ((size_t)(head_row0 + i * 128 + r)) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tmem + C::TM_DQ + lane_off + c * 32, v);
        tmem_ld_wait(v);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int cc = (u + lane) & 7;  // rotate to spread the rows' addresses
          atomicAdd(reinterpret_cast<float4*>(dst + c * 32 + cc * 4),
                    make_float4(__uint_as_float(v[cc * 4]), __uint_as_float(v[cc * 4 + 1]),
                                __uint_as_float(v[cc * 4 + 2]), __uint_as_float(v[cc * 4 + 3])));
        }
      }
      tc_fence_before();
      mbar_arrive(bar_tm_free);
    }
    if (ok) {
      ok = mbar_wait(bar_done, 0, abort_flag, kSiteBwdEpi);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      const size_t row = (size_t)(kv_row0 + r) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tmem + C::TM_DV + lane_off + c * 32, v);
        tmem_ld_wait(v);
        uint4* out = reinterpret_cast<uint4*>(args.dv + row + c * 32);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const float* f = reinterpret_cast<const float*>(&v[q4 * 8]);
          out[q4] = make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                               pack_bf16x2(f[6], f[7]));
        }
      }
      const float sc = args.scale;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tmem + C::TM_DK + lane_off + c * 32, v);
        tmem_ld_wait(v);
        uint4* out = reinterpret_cast<uint4*>(args.dk + row + c * 32);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const float* f = reinterpret_cast<const float*>(&v[q4 * 8]);
          out[q4] = make_uint4(pack_bf16x2(f[0] * sc, f[1] * sc), pack_bf16x2(f[2] * sc, f[3] * sc),
                               pack_bf16x2(f[4] * sc, f[5] * sc), pack_bf16x2(f[6] * sc, f[7] * sc));
        }
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace fattn
