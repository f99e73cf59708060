// fwd_kernel.cuh -- fused exact-attention forward for sm_100a.
//
// One CTA owns one 128-row query tile of one (batch, head).  It streams the
// 128-row key/value tiles of that head through a shared-memory ring and keeps
// the running row max m and row sum l of the online softmax in registers, so
// the N x N score matrix never leaves the chip (page 2 "一、用分块计算提高片上
// 数据复用" and "二、在线 Softmax 保持精确结果"; page 3 "4.1 分块计算" and "4.2
// 在线softmax技巧").  Only O and the per-row log-sum-exp are written (page 2
// "三、融合算子减少中间张量落盘").
//
// Roles (256 threads, warp-specialised):
//   warp 0      TMA producer: Q once, then K_j, V_j into an NSLOT-deep ring.
//   warp 1      tcgen05 issuer (one thread): S_j = Q K_j^T into one of two TMEM
//               score buffers; O += P_{j-1} V_{j-1} into the TMEM accumulator.
//   warps 4..7  softmax warpgroup, thread = query row: reads S_j from TMEM,
//               applies scale, mask and the online-softmax update, rescales
//               the O accumulator when the row max grows, writes P_j (bf16)
//               into swizzled shared memory; epilogue O / l -> bf16 -> TMA store.
//
// Tensor memory (512 columns x 128 lanes): S buffers at columns 0 and 128,
// O accumulator at column 256 (D columns).
#pragma once

#include "sm100.cuh"

namespace fattn {

struct FwdArgs {
  float* lse;         // [B*H*N] fp32
  int N;              // keys per head (multiple of 128)
  int num_q_tiles;    // N / 128
  float scale_log2;   // scale * log2(e)
};

template <int D>
struct FwdCfg {
  static constexpr int BM = 128;
  static constexpr int BN = 128;
  static constexpr int KB = D / 64;                    // 128-byte k-blocks per row
  static constexpr int TILE = 128 * D * 2;             // bytes of one Q/K/V tile
  static constexpr int NSLOT = (D == 128) ? 4 : 6;     // K/V ring depth
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_SLOT = TILE;
  static constexpr int OFF_P = OFF_SLOT + NSLOT * TILE;
  static constexpr int P_BYTES = 128 * 128 * 2;
  static constexpr int OFF_BAR = OFF_P + P_BYTES;
  // barriers: q_full, slot_full[NSLOT], slot_empty[NSLOT], s_full[2], s_free[2], p_full, o_done, drain
  static constexpr int NBAR = 1 + 2 * NSLOT + 4 + 3;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;  // tmem base (4 B), abort flag (4 B)
  static constexpr int SMEM = OFF_MISC + 16 + 1024;    // + slack for 1024-byte alignment
  static constexpr int TMEM_COLS = 512;
  static constexpr int TM_S0 = 0, TM_S1 = 128, TM_O = 256;
};

enum : int {  // wait sites recorded in the device status word on a timeout
  kSiteFwdProducer = 0x101,
  kSiteFwdMmaQ = 0x102,
  kSiteFwdMmaK = 0x103,
  kSiteFwdMmaS = 0x104,
  kSiteFwdMmaP = 0x105,
  kSiteFwdMmaV = 0x106,
  kSiteFwdSoftS = 0x107,
  kSiteFwdSoftO = 0x108,
};

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(256, 1)
    fattn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                     const FwdArgs args) {
  using C = FwdCfg<D>;
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);

  const uint32_t sQ = sbase + C::OFF_Q;
  const uint32_t sSlot0 = sbase + C::OFF_SLOT;
  const uint32_t sP = sbase + C::OFF_P;
  const uint32_t bar0 = sbase + C::OFF_BAR;
  const uint32_t bar_q_full = bar0;
  auto bar_slot_full = [&](int s) { return bar0 + 8u * (1 + s); };
  auto bar_slot_empty = [&](int s) { return bar0 + 8u * (1 + C::NSLOT + s); };
  auto bar_s_full = [&](int b) { return bar0 + 8u * (1 + 2 * C::NSLOT + b); };
  auto bar_s_free = [&](int b) { return bar0 + 8u * (3 + 2 * C::NSLOT + b); };
  const uint32_t bar_p_full = bar0 + 8u * (5 + 2 * C::NSLOT);
  const uint32_t bar_o_done = bar0 + 8u * (6 + 2 * C::NSLOT);
  const uint32_t bar_drain = bar0 + 8u * (7 + 2 * C::NSLOT);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Work unit: the query tile varies fastest so that the CTAs resident at one
  // time share a head's K/V in L2; causal heads run their longest tiles first.
  const int NT = args.num_q_tiles;
  const int bh = (int)(blockIdx.x / (unsigned)NT);
  const int t_in_head = (int)(blockIdx.x % (unsigned)NT);
  const int q_tile = CAUSAL ? (NT - 1 - t_in_head) : t_in_head;
  const int head_row0 = bh * args.N;
  const int q_row0 = head_row0 + q_tile * C::BM;
  const int n_kv = CAUSAL ? (q_tile + 1) : NT;

  if (threadIdx.x == 0) {
    mbar_init(bar_q_full, 1);
    for (int s = 0; s < C::NSLOT; ++s) {
      mbar_init(bar_slot_full(s), 1);
      mbar_init(bar_slot_empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_s_full(b), 1);
      mbar_init(bar_s_free(b), 128);
    }
    mbar_init(bar_p_full, 128);
    mbar_init(bar_o_done, 1);
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
      prefetch_tensormap(&tm_o);
      mbar_arrive_expect_tx(bar_q_full, C::TILE);
#pragma unroll
      for (int kb = 0; kb < C::KB; ++kb) tma_load_2d(sQ + kb * 16384, &tm_q, bar_q_full, kb * 64, q_row0);
      int it = 0;
      bool ok = true;
      for (int j = 0; j < n_kv && ok; ++j) {
        for (int t = 0; t < 2; ++t, ++it) {
          const int s = it % C::NSLOT;
          const uint32_t use = it / C::NSLOT;
          if (!mbar_wait(bar_slot_empty(s), (use & 1) ^ 1, abort_flag, kSiteFwdProducer)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar_slot_full(s), C::TILE);
          const CUtensorMap* map = (t == 0) ? &tm_k : &tm_v;
          const uint32_t dst = sSlot0 + s * C::TILE;
#pragma unroll
          for (int kb = 0; kb < C::KB; ++kb)
            tma_load_2d(dst + kb * 16384, map, bar_slot_full(s), kb * 64, head_row0 + j * C::BN);
        }
      }
      if (!ok) {
        // Abort: let the copies already issued land before the CTA exits.
        mbar_wait_ns(bar_q_full, 0, 100000000ull);
        for (int i = (it > C::NSLOT ? it - C::NSLOT : 0); i < it; ++i)
          mbar_wait_ns(bar_slot_full(i % C::NSLOT), (i / C::NSLOT) & 1, 100000000ull);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, 128, false, false);  // Q (K-major) x K (K-major)
      constexpr uint32_t idPV = idesc_bf16_f32(128, D, false, true);    // P (K-major) x V (MN-major)
      bool ok = mbar_wait(bar_q_full, 0, abort_flag, kSiteFwdMmaQ);
      tc_fence_after();
      auto issue_pv = [&](int jj) -> bool {
        const int it = 2 * jj + 1;
        const int s = it % C::NSLOT;
        if (!mbar_wait(bar_slot_full(s), (it / C::NSLOT) & 1, abort_flag, kSiteFwdMmaV)) return false;
        if (!mbar_wait(bar_p_full, jj & 1, abort_flag, kSiteFwdMmaP)) return false;
        tc_fence_after();
        const uint32_t sV = sSlot0 + s * C::TILE;
#pragma unroll
        for (int kk = 0; kk < C::BN / 16; ++kk) {
          const uint64_t a = sdesc_sw128(sP + (kk >> 2) * 16384 + (kk & 3) * 32, 16);
          const uint64_t b = sdesc_sw128(sV + kk * 2048, 16384);
          mma_ss(tmem + C::TM_O, a, b, idPV, (jj > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(bar_o_done);
        mma_commit(bar_slot_empty(s));
        return true;
      };
      for (int j = 0; j < n_kv && ok; ++j) {
        const int it = 2 * j;
        const int s = it % C::NSLOT;
        const int sb = j & 1;
        if (!mbar_wait(bar_slot_full(s), (it / C::NSLOT) & 1, abort_flag, kSiteFwdMmaK)) {
          ok = false;
          break;
        }
        if (!mbar_wait(bar_s_free(sb), ((j >> 1) & 1) ^ 1, abort_flag, kSiteFwdMmaS)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sK = sSlot0 + s * C::TILE;
        const uint32_t tS = tmem + (sb ? C::TM_S1 : C::TM_S0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t a = sdesc_sw128(sQ + (kk >> 2) * 16384 + (kk & 3) * 32, 16);
          const uint64_t b = sdesc_sw128(sK + (kk >> 2) * 16384 + (kk & 3) * 32, 16);
          mma_ss(tS, a, b, idS, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar_s_full(sb));
        mma_commit(bar_slot_empty(s));
        if (j > 0 && !issue_pv(j - 1)) ok = false;
      }
      if (ok) ok = issue_pv(n_kv - 1);
      // Make sure nothing this thread issued is still running before TMEM is freed.
      mma_commit(bar_drain);
      mbar_wait_ns(bar_drain, 0, 100000000ull);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------ softmax warpgroup
    const int wq = warp - 4;
    const int r = wq * 32 + lane;                 // row inside the query tile
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const float sl2 = args.scale_log2;
    float m = -INFINITY;  // running max of the scaled scores, log2 units
    float l = 0.f;        // running sum of exp2(score - m)
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const int sb = j & 1;
      ok = mbar_wait(bar_s_full(sb), (j >> 1) & 1, abort_flag, kSiteFwdSoftS);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      float s[128];
      const uint32_t tS = tmem + (sb ? C::TM_S1 : C::TM_S0) + lane_off;
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        uint32_t v[32];
        tmem_ld32(tS + c4 * 32, v);
        tmem_ld_wait(v);
#pragma unroll
        for (int i = 0; i < 32; ++i) s[c4 * 32 + i] = __uint_as_float(v[i]) * sl2;
      }
      tc_fence_before();
      mbar_arrive(bar_s_free(sb));
      if (CAUSAL && j == q_tile) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c > r) s[c] = -INFINITY;
      }
      float mx = m;
#pragma unroll
      for (int c = 0; c < 128; ++c) mx = fmaxf(mx, s[c]);
      const float alpha = ex2(m - mx);
      float sum = 0.f;
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        s[c] = ex2(s[c] - mx);
        sum += s[c];
      }
      l = l * alpha + sum;
      m = mx;
      if (j > 0) {
        // P_{j-1} V_{j-1} must be finished: it frees the P buffer and makes O stable.
        ok = mbar_wait(bar_o_done, (j - 1) & 1, abort_flag, kSiteFwdSoftO);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        if (__any_sync(0xffffffffu, alpha != 1.f)) {
          const uint32_t tO = tmem + C::TM_O + lane_off;
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t v[32];
            tmem_ld32(tO + c * 32, v);
            tmem_ld_wait(v);
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * alpha);
            tmem_st32(tO + c * 32, v);
          }
          tmem_st_wait();
        }
      }
      // P (bf16) -> shared memory, K-major 128B-swizzled, two 64-column blocks.
#pragma unroll
      for (int ch = 0; ch < 16; ++ch) {
        const int c0 = ch * 8;
        const uint32_t addr = sP + (ch >> 3) * 16384 + sw128_offset(r, ch & 7);
        st_shared_v4(addr, pack_bf16x2(s[c0], s[c0 + 1]), pack_bf16x2(s[c0 + 2], s[c0 + 3]),
                     pack_bf16x2(s[c0 + 4], s[c0 + 5]), pack_bf16x2(s[c0 + 6], s[c0 + 7]));
      }
      fence_async_shared();
      tc_fence_before();
      mbar_arrive(bar_p_full);
    }
    if (ok) {
      ok = mbar_wait(bar_o_done, (n_kv - 1) & 1, abort_flag, kSiteFwdSoftO);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.f / l;
      const uint32_t tO = tmem + C::TM_O + lane_off;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tO + c * 32, v);
        tmem_ld_wait(v);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const int chunk = (c & 1) * 4 + q4;
          const uint32_t addr = sQ + (c >> 1) * 16384 + sw128_offset(r, chunk);
          const float* f = reinterpret_cast<const float*>(&v[q4 * 8]);
          st_shared_v4(addr, pack_bf16x2(f[0] * inv_l, f[1] * inv_l), pack_bf16x2(f[2] * inv_l, f[3] * inv_l),
                       pack_bf16x2(f[4] * inv_l, f[5] * inv_l), pack_bf16x2(f[6] * inv_l, f[7] * inv_l));
        }
      }
      // natural-log LSE of the scaled scores: (m + log2 l) * ln 2
      args.lse[q_row0 + r] = (m + __log2f(l)) * 0.69314718055994530942f;
      fence_async_shared();
      named_barrier(1, 128);
      if (r == 0) {
#pragma unroll
        for (int kb = 0; kb < C::KB; ++kb) tma_store_2d(&tm_o, sQ + kb * 16384, kb * 64, q_row0);
        bulk_commit();
        bulk_wait0();
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
