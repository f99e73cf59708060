// bwd_kernels.cuh -- exact-attention backward for sm_100a.
//
// The backward recomputes S and P tile by tile from Q, K and the saved
// log-sum-exp instead of reading a stored probability matrix (page 2 "四、反向
// 传播选择重计算而非全量保存").  Three kernels run in order on one stream:
//
//  1. fattn_bwd_pre_kernel   D_i = sum_c dO_ic O_ic, LSE2_i = LSE_i log2(e),
//                            and zero the fp32 dQ accumulator.     (HBM-bound)
//  2. fattn_bwd_dkdv_kernel  one CTA per (batch*head, 128-row key tile j);
//                            loops over the 64-row query sub-tiles i that can
//                            see tile j and, on the tcgen05 tensor cores,
//                              S^T  = K_j Q_i^T          (TMEM, two buffers)
//                              dP^T = V_j dO_i^T         (TMEM)
//                              P^T  = exp2(S^T scale log2e - LSE2_i)   (masked)
//                              dS^T = P^T o (dP^T - D_i)
//                              dV_j += P^T dO_i   (P^T read from TMEM)
//                              dK_j += dS^T Q_i   (dS^T read from TMEM)
//                              dQ_i^T = K_j^T dS^T_i -> fp32 atomics into the
//                                                       accumulator
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
  const float* lse2;  // [B*H*N]  LSE * log2(e)
  const float* dvec;  // [B*H*N]  D
  float* dq_acc;      // [B*H*N, D] fp32
  int N;
  int num_tiles;      // N / 128
  float scale;        // for dK
  float scale_log2;   // scale * log2(e)
};

template <int D>
struct BwdCfg {
  static constexpr int KB = D / 64;              // 64-column (128-byte) blocks per row
  static constexpr int BQ = 64;                  // query rows per inner step
  static constexpr int NS = 3;                   // Q/dO ring depth
  static constexpr int KV_TILE = 128 * D * 2;    // bytes of the K (or V) tile
  static constexpr int KV_BLK = 128 * 128;       // one 64-column block of a 128-row tile
  static constexpr int Q_TILE = BQ * D * 2;      // bytes of a Q (or dO) sub-tile
  static constexpr int Q_BLK = BQ * 128;         // one 64-column block of a 64-row sub-tile
  static constexpr int DS_BYTES = 128 * BQ * 2;  // dS^T [128 keys][64 queries] bf16
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = KV_TILE;
  static constexpr int OFF_STAGE = 2 * KV_TILE;
  static constexpr int STAGE = 2 * Q_TILE;       // Q sub-tile, then dO sub-tile
  static constexpr int OFF_DS = OFF_STAGE + NS * STAGE;
  static constexpr int OFF_STAT = OFF_DS + 2 * DS_BYTES;  // per stage: LSE2[64], D[64] fp32
  static constexpr int OFF_BAR = OFF_STAT + NS * 512;
  // kv_full, q_full[NS], q_empty[NS], st_full[2], ds_full[2], dq_full[2], dq_free[2], done, drain
  static constexpr int NBAR = 1 + 2 * NS + 8 + 2;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;
  static constexpr int TMEM_COLS = 512;
  // Two 128-column regions R_b: S^T at +0 (once read, P^T and dS^T as bf16
  // pairs overlay its columns 0..31 and 32..63), dP^T at +64 (dQ^T of the same
  // step replaces it once it has been read).  Then the dV and dK accumulators.
  static constexpr int TM_R0 = 0, TM_R1 = 128, TM_DV = 256, TM_DK = 256 + D;
};

enum : int {
  kSiteBwdProducer = 0x201,
  kSiteBwdMmaKV = 0x202,
  kSiteBwdMmaQ = 0x203,
  kSiteBwdMmaDS = 0x205,
  kSiteBwdMmaDQ = 0x206,
  kSiteBwdSoftS = 0x207,
  kSiteBwdSoftQ = 0x208,
  kSiteBwdDrain = 0x209,
  kSiteBwdEpi = 0x20a,
};

// Roles (320 threads):
//   warps 0..3  softmax-gradient group, thread = key row of the tile: P^T, dS^T
//   warps 4..7  dQ drain (thread = head-dim lane of dQ^T) and the dK/dV epilogue
//   warp 8      TMA producer (K, V once; Q/dO sub-tiles through an NS-deep ring)
//   warp 9      tcgen05 issuer (one thread)
template <int D, bool CAUSAL>
__global__ void __launch_bounds__(320, 1)
    fattn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                          const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
                          const BwdArgs args) {
  using C = BwdCfg<D>;
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const uint32_t sK = sbase + C::OFF_K, sV = sbase + C::OFF_V;
  auto sQ = [&](int s) { return sbase + C::OFF_STAGE + s * C::STAGE; };
  auto sDO = [&](int s) { return sbase + C::OFF_STAGE + s * C::STAGE + C::Q_TILE; };
  auto sDS = [&](int b) { return sbase + C::OFF_DS + b * C::DS_BYTES; };
  auto sStat = [&](int s) { return sbase + C::OFF_STAT + s * 512; };
  auto stat = [&](int s) { return reinterpret_cast<const float*>(smem + C::OFF_STAT + s * 512); };
  const uint32_t bar0 = sbase + C::OFF_BAR;
  const uint32_t bar_kv_full = bar0;
  auto bar_q_full = [&](int s) { return bar0 + 8u * (1 + s); };
  auto bar_q_empty = [&](int s) { return bar0 + 8u * (1 + C::NS + s); };
  auto bar_st_full = [&](int b) { return bar0 + 8u * (1 + 2 * C::NS + b); };
  auto bar_ds_full = [&](int b) { return bar0 + 8u * (3 + 2 * C::NS + b); };
  auto bar_dq_full = [&](int b) { return bar0 + 8u * (5 + 2 * C::NS + b); };
  auto bar_dq_free = [&](int b) { return bar0 + 8u * (7 + 2 * C::NS + b); };
  const uint32_t bar_done = bar0 + 8u * (9 + 2 * C::NS);
  const uint32_t bar_drain = bar0 + 8u * (10 + 2 * C::NS);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int NT = args.num_tiles;
  // The key tile varies fastest so that the CTAs resident at one time add into
  // the same head's dQ rows (which then stay in L2); causal: tile 0 sees the most
  // query rows and is launched first.
  const int bh = (int)(blockIdx.x / (unsigned)NT);
  const int kv_tile = (int)(blockIdx.x % (unsigned)NT);
  const int head_row0 = bh * args.N;
  const int kv_row0 = head_row0 + kv_tile * 128;
  const int q_begin = CAUSAL ? kv_tile * 128 : 0;  // first query row (in the head) that sees this tile
  const int n_it = (args.N - q_begin) / C::BQ;

  if (threadIdx.x == 0) {
    mbar_init(bar_kv_full, 1);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(bar_q_full(s), 1);
      mbar_init(bar_q_empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_st_full(b), 1);
      mbar_init(bar_ds_full(b), 128);
      mbar_init(bar_dq_full(b), 1);
      mbar_init(bar_dq_free(b), 128);
    }
    mbar_init(bar_done, 1);
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_addr(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
      prefetch_tensormap(&tm_do);
      mbar_arrive_expect_tx(bar_kv_full, 2 * C::KV_TILE);
#pragma unroll
      for (int kb = 0; kb < C::KB; ++kb) {
        tma_load_2d(sK + kb * C::KV_BLK, &tm_k, bar_kv_full, kb * 64, kv_row0);
        tma_load_2d(sV + kb * C::KV_BLK, &tm_v, bar_kv_full, kb * 64, kv_row0);
      }
      int it = 0;
      for (; it < n_it; ++it) {
        const int s = it % C::NS;
        if (!mbar_wait(bar_q_empty(s), ((it / C::NS) & 1) ^ 1, abort_flag, kSiteBwdProducer)) break;
        const int q_row = head_row0 + q_begin + it * C::BQ;
        mbar_arrive_expect_tx(bar_q_full(s), C::STAGE + 512);
#pragma unroll
        for (int kb = 0; kb < C::KB; ++kb) {
          tma_load_2d(sQ(s) + kb * C::Q_BLK, &tm_q, bar_q_full(s), kb * 64, q_row);
          tma_load_2d(sDO(s) + kb * C::Q_BLK, &tm_do, bar_q_full(s), kb * 64, q_row);
        }
        bulk_load(sStat(s), args.lse2 + q_row, 256, bar_q_full(s));
        bulk_load(sStat(s) + 256, args.dvec + q_row, 256, bar_q_full(s));
      }
      if (it < n_it) {  // aborted: let the copies already issued land
        mbar_wait_ns(bar_kv_full, 0, 100000000ull);
        for (int i = (it > C::NS ? it - C::NS : 0); i < it; ++i)
          mbar_wait_ns(bar_q_full(i % C::NS), (i / C::NS) & 1, 100000000ull);
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    // ----------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_bf16_f32(128, C::BQ, false, false);  // K/V (K-major) x Q/dO (K-major)
      constexpr uint32_t id_kv = idesc_bf16_f32(128, D, false, true);      // P^T|dS^T (K-major) x dO|Q (MN)
      constexpr uint32_t id_q = idesc_bf16_f32(128, C::BQ, true, true);    // K^T (MN) x dS^T (MN)
      // For d = 64 the dQ^T product still uses M = 128: the second 64-row half of
      // A repeats the first (LBO = 0) and its output lanes are ignored.
      constexpr uint32_t kt_lbo = (D == 128) ? C::KV_BLK : 0;
      bool ok = mbar_wait(bar_kv_full, 0, abort_flag, kSiteBwdMmaKV);
      auto region = [&](int b) { return tmem + (b ? C::TM_R1 : C::TM_R0); };
      auto issue_s_dp = [&](int it) -> bool {  // S^T, dP^T of step `it` into region it % 2
        const int s = it % C::NS;
        if (!mbar_wait(bar_q_full(s), (it / C::NS) & 1, abort_flag, kSiteBwdMmaQ)) return false;
        tc_fence_after();
        const uint32_t R = region(it & 1);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ka = (kk >> 2) * C::KV_BLK + (kk & 3) * 32;
          const uint32_t kb = (kk >> 2) * C::Q_BLK + (kk & 3) * 32;
          mma_ss(R, sdesc_sw128(sK + ka, 16), sdesc_sw128(sQ(s) + kb, 16), id_s, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ka = (kk >> 2) * C::KV_BLK + (kk & 3) * 32;
          const uint32_t kb = (kk >> 2) * C::Q_BLK + (kk & 3) * 32;
          mma_ss(R + 64, sdesc_sw128(sV + ka, 16), sdesc_sw128(sDO(s) + kb, 16), id_s, kk > 0);
        }
        mma_commit(bar_st_full(it & 1));
        return true;
      };
      // Tensor-core order: S,dP(0) S,dP(1) | dV,dK,dQ(0) S,dP(2) | dV,dK,dQ(1) S,dP(3) | ...
      // so that the softmax-gradient group works on step i+1 while the tensor
      // cores run the five products of steps i and i+2.
      if (ok) ok = issue_s_dp(0);
      if (ok && n_it > 1) ok = issue_s_dp(1);
      for (int it = 0; it < n_it && ok; ++it) {
        const int s = it % C::NS, b = it & 1;
        if (!(ok = mbar_wait(bar_ds_full(b), (it >> 1) & 1, abort_flag, kSiteBwdMmaDS))) break;
        tc_fence_after();
        const uint32_t R = region(b);
        // dV += P^T dO  (A = P^T from TMEM: 4 x 16 query columns, 8 TMEM columns each)
#pragma unroll
        for (int kk = 0; kk < C::BQ / 16; ++kk)
          mma_ts(tmem + C::TM_DV, R + kk * 8, sdesc_sw128(sDO(s) + kk * 2048, C::Q_BLK), id_kv,
                 (it > 0 || kk > 0) ? 1u : 0u);
        // dK += dS^T Q  (A = dS^T from TMEM, columns 32..63 of the region)
#pragma unroll
        for (int kk = 0; kk < C::BQ / 16; ++kk)
          mma_ts(tmem + C::TM_DK, R + 32 + kk * 8, sdesc_sw128(sQ(s) + kk * 2048, C::Q_BLK), id_kv,
                 (it > 0 || kk > 0) ? 1u : 0u);
        mma_commit(bar_q_empty(s));
        // dQ^T = K^T dS^T into the dP^T half of this region (already read)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(R + 64, sdesc_sw128(sK + kk * 2048, kt_lbo), sdesc_sw128(sDS(b) + kk * 2048, 16), id_q,
                 kk > 0 ? 1u : 0u);
        mma_commit(bar_dq_full(b));
        if (it + 2 < n_it) {
          // region b is free once dQ^T(it) has been drained (which also implies that
          // dV(it), the reader of P^T, has completed)
          if (!(ok = mbar_wait(bar_dq_free(b), (it >> 1) & 1, abort_flag, kSiteBwdMmaDQ))) break;
          if (!(ok = issue_s_dp(it + 2))) break;
        }
      }
      if (ok) mma_commit(bar_done);
      mma_commit(bar_drain);
      mbar_wait_ns(bar_drain, 0, 100000000ull);
    }
    __syncwarp();
  } else if (warp < 4) {
    // ------------------------------------------------- softmax-gradient group
    const int r = warp * 32 + lane;  // key row inside the tile
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const int kv_idx = kv_tile * 128 + r;
    const float sl2 = args.scale_log2;
    for (int it = 0; it < n_it; ++it) {
      const int s = it % C::NS, b = it & 1;
      bool ok = mbar_wait(bar_st_full(b), (it >> 1) & 1, abort_flag, kSiteBwdSoftS);
      ok = ok && mbar_wait(bar_q_full(s), (it / C::NS) & 1, abort_flag, kSiteBwdSoftQ);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const uint32_t tS = tmem + (b ? C::TM_R1 : C::TM_R0) + lane_off;
      const float* lse_s = stat(s);
      const float* dvec_s = stat(s) + 64;
      const int q0 = q_begin + it * C::BQ;  // first query row (in the head) of this sub-tile
      const bool diag = CAUSAL && (q0 < kv_tile * 128 + 128);
      uint32_t pk[32];   // P^T row, packed bf16 pairs
      uint32_t dsk[32];  // dS^T row, packed bf16 pairs
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t sv[32], dv[32];
        tmem_ld32(tS + h * 32, sv);
        tmem_ld_wait(sv);
        tmem_ld32(tS + 64 + h * 32, dv);
        tmem_ld_wait(dv);
        float ds[32];
#pragma unroll
        for (int t = 0; t < 32; ++t) {
          const int c = h * 32 + t;
          float p = ex2(fmaf(__uint_as_float(sv[t]), sl2, -lse_s[c]));
          if (diag && (q0 + c) < kv_idx) p = 0.f;
          ds[t] = p * (__uint_as_float(dv[t]) - dvec_s[c]);
          sv[t] = __float_as_uint(p);
        }
#pragma unroll
        for (int t = 0; t < 16; ++t) {
          pk[h * 16 + t] = pack_bf16x2(__uint_as_float(sv[2 * t]), __uint_as_float(sv[2 * t + 1]));
          dsk[h * 16 + t] = pack_bf16x2(ds[2 * t], ds[2 * t + 1]);
        }
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const int ch = h * 4 + q4;  // 16-byte chunk along the 64 query columns
          const uint32_t* w = &dsk[h * 16 + q4 * 4];
          st_shared_v4(sDS(b) + sw128_offset(r, ch), w[0], w[1], w[2], w[3]);
        }
      }
      tmem_st32(tS, pk);        // P^T (bf16) over columns 0..31 of this region
      tmem_st32(tS + 32, dsk);  // dS^T (bf16) over columns 32..63 (S^T already read)
      tmem_st_wait();
      fence_async_shared();
      tc_fence_before();
      mbar_arrive(bar_ds_full(b));
    }
    tc_fence_before();
  } else if (warp < 8) {
    // --------------------------------------------- dQ drain, dK/dV epilogue
    const int wq = warp - 4;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const bool has_d = wq * 32 < D;  // TMEM lane = head-dim index of dQ^T
    const int dcol = wq * 32 + lane;
    bool ok = true;
    for (int it = 0; it < n_it; ++it) {
      const int b = it & 1;
      ok = mbar_wait(bar_dq_full(b), (it >> 1) & 1, abort_flag, kSiteBwdDrain);
      if (!(ok = __all_sync(0xffffffffu, ok))) break;
      tc_fence_after();
      const uint32_t tDQ = tmem + (b ? C::TM_R1 : C::TM_R0) + 64 + lane_off;
      uint32_t v0[32], v1[32];
      if (has_d) {
        tmem_ld32(tDQ, v0);
        tmem_ld32(tDQ + 32, v1);
        tmem_ld_wait(v0);
        tmem_ld_wait(v1);
      }
      tc_fence_before();
      mbar_arrive(bar_dq_free(b));
      if (has_d) {
        float* dst = args.dq_acc + (size_t)(head_row0 + q_begin + it * C::BQ) * D + dcol;
#pragma unroll
        for (int c = 0; c < 32; ++c) atomicAdd(dst + (size_t)c * D, __uint_as_float(v0[c]));
#pragma unroll
        for (int c = 0; c < 32; ++c) atomicAdd(dst + (size_t)(32 + c) * D, __uint_as_float(v1[c]));
      }
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_done, 0, abort_flag, kSiteBwdEpi));
    if (ok) {
      tc_fence_after();
      // dV, dK rows (thread = key row) -> bf16 -> the now idle V and K tiles -> TMA store
      const int row = wq * 32 + lane;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint32_t tsrc = tmem + (which ? C::TM_DK : C::TM_DV) + lane_off;
        const uint32_t sdst = which ? sK : sV;
        const float mul = which ? args.scale : 1.f;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tsrc + c * 32, v);
          tmem_ld_wait(v);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const int chunk = (c & 1) * 4 + q4;
            const uint32_t* w = &v[q4 * 8];
            st_shared_v4(sdst + (c >> 1) * C::KV_BLK + sw128_offset(row, chunk),
                         pack_bf16x2(__uint_as_float(w[0]) * mul, __uint_as_float(w[1]) * mul),
                         pack_bf16x2(__uint_as_float(w[2]) * mul, __uint_as_float(w[3]) * mul),
                         pack_bf16x2(__uint_as_float(w[4]) * mul, __uint_as_float(w[5]) * mul),
                         pack_bf16x2(__uint_as_float(w[6]) * mul, __uint_as_float(w[7]) * mul));
          }
        }
      }
      fence_async_shared();
      named_barrier(1, 128);
      if (wq == 0 && lane == 0) {
#pragma unroll
        for (int kb = 0; kb < C::KB; ++kb) {
          tma_store_2d(&tm_dv, sV + kb * C::KV_BLK, kb * 64, kv_row0);
          tma_store_2d(&tm_dk, sK + kb * C::KV_BLK, kb * 64, kv_row0);
        }
        bulk_commit();
        bulk_wait0();
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace fattn
