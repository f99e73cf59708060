// fwd_kernel.cuh -- fused exact-attention forward for sm_100a.
//
// One CTA owns two consecutive 128-row query tiles of one (batch, head).  It
// streams the 128-row key/value tiles of that head through a shared-memory ring
// and keeps the running row max m and row sum l of the online softmax in
// registers, so the N x N score matrix never leaves the chip (page 2 "一、用分块
// 计算提高片上数据复用" and "二、在线 Softmax 保持精确结果"; page 3 "4.1 分块计算"
// and "4.2 在线softmax技巧").  Only O and the per-row log-sum-exp are written
// (page 2 "三、融合算子减少中间张量落盘").
//
// Roles (384 threads = three warpgroups, warp-specialised):
//   warps 0..3  softmax group 0, thread = row of query tile 0   (224 registers)
//   warps 4..7  softmax group 1, thread = row of query tile 1   (224 registers)
//   warp 8      TMA producer: Q0, Q1 once, then K_j, V_j through an NSLOT-deep ring
//   warp 9      tcgen05 issuer (one thread); warps 10, 11 idle   (56 registers)
//                 S0 = Q0 K_j^T, S1 = Q1 K_j^T          (TMEM, fp32)
//                 O0 += P0 V_j,  O1 += P1 V_j           (P read from TMEM)
// While group 0 turns S0 into P0 the tensor cores compute S1 (and vice versa),
// so the exponentials of one tile overlap the products of the other.
//
// Tensor memory (512 columns x 128 lanes): S0 at column 0, S1 at 128 (P_k, bf16,
// overlays the first 64 columns of S_k), O0 at 256, O1 at 256 + D.
//
// Online softmax with a lazily updated reference max: each row keeps a
// reference m_ref (log2 units) and sums exp2(s - m_ref).  When a tile's row max
// exceeds m_ref by more than kRescaleThreshold, m_ref moves up and the partial
// O and l are multiplied by exp2(m_old - m_new) (page 2: "按照新的数值尺度修正此
// 前的累加结果").  Otherwise m_ref stays, weights stay <= 2^threshold, and since O
// and l share the same reference the final O / l is unchanged.
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
  static constexpr int KB = D / 64;                 // 128-byte column blocks per row
  static constexpr int TILE = 128 * D * 2;          // bytes of one 128-row Q/K/V tile
  static constexpr int BLK = 128 * 128;             // one 64-column block of a tile
  static constexpr int NSLOT = (D == 128) ? 4 : 6;  // K/V ring depth
  static constexpr int OFF_Q = 0;                   // Q0, Q1 (reused for the O epilogue)
  static constexpr int OFF_SLOT = 2 * TILE;
  static constexpr int OFF_BAR = OFF_SLOT + NSLOT * TILE;
  // q_full, slot_full[NSLOT], slot_empty[NSLOT], s_full[2], p_full[2], pv_done[2], drain
  static constexpr int NBAR = 1 + 2 * NSLOT + 6 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;  // tmem base (4 B), abort flag (4 B)
  static constexpr int SMEM = OFF_MISC + 16 + 1024;    // + slack for 1024-byte alignment
  static constexpr int TMEM_COLS = 512;
  static constexpr int TM_S = 0;                       // S_k at k * 128
  static constexpr int TM_O = 256;                     // O_k at 256 + k * D
};

constexpr float kRescaleThreshold = 8.0f;  // log2 units: weights stay below 256
// Exponentials evaluated on the FMA pipe (exp2_poly_x2) per 8 pairs of columns;
// the rest use MUFU ex2.  On B200 at this tile shape the extra FMA-pipe
// instructions cost about what they save on MUFU, so the share is 0.
constexpr int kPolyPairsPer8 = 0;

enum : int {  // wait sites recorded in the device status word on a timeout
  kSiteFwdProducer = 0x101,
  kSiteFwdMmaQ = 0x102,
  kSiteFwdMmaK = 0x103,
  kSiteFwdMmaPV = 0x104,
  kSiteFwdMmaP = 0x105,
  kSiteFwdMmaV = 0x106,
  kSiteFwdSoftS = 0x107,
  kSiteFwdSoftO = 0x108,
};

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(384, 1)
    fattn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                     const FwdArgs args) {
  using C = FwdCfg<D>;
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);

  auto sQ = [&](int k) { return sbase + C::OFF_Q + k * C::TILE; };
  const uint32_t sSlot0 = sbase + C::OFF_SLOT;
  const uint32_t bar0 = sbase + C::OFF_BAR;
  const uint32_t bar_q_full = bar0;
  auto bar_slot_full = [&](int s) { return bar0 + 8u * (1 + s); };
  auto bar_slot_empty = [&](int s) { return bar0 + 8u * (1 + C::NSLOT + s); };
  auto bar_s_full = [&](int k) { return bar0 + 8u * (1 + 2 * C::NSLOT + k); };
  auto bar_p_full = [&](int k) { return bar0 + 8u * (3 + 2 * C::NSLOT + k); };
  auto bar_pv_done = [&](int k) { return bar0 + 8u * (5 + 2 * C::NSLOT + k); };
  const uint32_t bar_drain = bar0 + 8u * (7 + 2 * C::NSLOT);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Work unit: a pair of query tiles; the pair index varies fastest so that the
  // CTAs resident at one time share a head's K/V in L2.  Causal heads start with
  // their longest pairs.
  const int NT = args.num_q_tiles;
  const int NP = (NT + 1) >> 1;
  const int bh = (int)(blockIdx.x / (unsigned)NP);
  const int p_in_head = (int)(blockIdx.x % (unsigned)NP);
  const int pair = CAUSAL ? (NP - 1 - p_in_head) : p_in_head;
  const int head_row0 = bh * args.N;
  const int tile0 = 2 * pair;
  const bool has_q1 = tile0 + 1 < NT;
  // key tiles each query tile needs (contiguous from 0)
  const int n_kv0 = CAUSAL ? tile0 + 1 : NT;
  const int n_kv1 = has_q1 ? (CAUSAL ? tile0 + 2 : NT) : 0;
  const int n_kv = n_kv1 > n_kv0 ? n_kv1 : n_kv0;

  if (threadIdx.x == 0) {
    mbar_init(bar_q_full, 1);
    for (int s = 0; s < C::NSLOT; ++s) {
      mbar_init(bar_slot_full(s), 1);
      mbar_init(bar_slot_empty(s), 1);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(bar_s_full(k), 1);
      mbar_init(bar_p_full(k), 128);
      mbar_init(bar_pv_done(k), 1);
    }
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

  // 384 threads launch with 168 registers each (64512 in all); the softmax groups
  // take 224, the producer/MMA group keeps 56: 2*128*224 + 128*56 = 64512.
  if (warp >= 8) {
    regs_decrease<56>();
    if (warp == 8) {
      // ------------------------------------------------------------ producer
      if (lane == 0) {
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
        prefetch_tensormap(&tm_o);
        mbar_arrive_expect_tx(bar_q_full, (has_q1 ? 2 : 1) * C::TILE);
        for (int k = 0; k < (has_q1 ? 2 : 1); ++k)
  #pragma unroll
          for (int kb = 0; kb < C::KB; ++kb)
            tma_load_2d(sQ(k) + kb * C::BLK, &tm_q, bar_q_full, kb * 64, head_row0 + (tile0 + k) * 128);
        int it = 0;
        bool ok = true;
        for (int j = 0; j < n_kv && ok; ++j) {
          for (int t = 0; t < 2; ++t, ++it) {
            const int s = it % C::NSLOT;
            if (!mbar_wait(bar_slot_empty(s), ((it / C::NSLOT) & 1) ^ 1, abort_flag, kSiteFwdProducer)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(bar_slot_full(s), C::TILE);
            const CUtensorMap* map = (t == 0) ? &tm_k : &tm_v;
            const uint32_t dst = sSlot0 + s * C::TILE;
  #pragma unroll
            for (int kb = 0; kb < C::KB; ++kb)
              tma_load_2d(dst + kb * C::BLK, map, bar_slot_full(s), kb * 64, head_row0 + j * 128);
          }
        }
        if (!ok) {  // aborted: let the copies already issued land before the CTA exits
          mbar_wait_ns(bar_q_full, 0, 100000000ull);
          for (int i = (it > C::NSLOT ? it - C::NSLOT : 0); i < it; ++i)
            mbar_wait_ns(bar_slot_full(i % C::NSLOT), (i / C::NSLOT) & 1, 100000000ull);
        }
      }
      __syncwarp();
    } else if (warp == 9) {
      // ----------------------------------------------------------- MMA issuer
      if (lane == 0) {
        constexpr uint32_t idS = idesc_bf16_f32(128, 128, false, false);  // Q (K-major) x K (K-major)
        constexpr uint32_t idPV = idesc_bf16_f32(128, D, false, true);    // P (TMEM) x V (MN-major)
        bool ok = mbar_wait(bar_q_full, 0, abort_flag, kSiteFwdMmaQ);
        auto act = [&](int k, int j) { return j < (k == 0 ? n_kv0 : n_kv1); };
        auto slot_of = [&](int it) { return it % C::NSLOT; };
        auto issue_s = [&](int k, int j) {  // S_k = Q_k K_j^T
          const uint32_t kaddr = sSlot0 + slot_of(2 * j) * C::TILE;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * C::BLK + (kk & 3) * 32;
            mma_ss(tmem + C::TM_S + k * 128, sdesc_sw128(sQ(k) + off, 16), sdesc_sw128(kaddr + off, 16), idS,
                   kk > 0 ? 1u : 0u);
          }
          mma_commit(bar_s_full(k));
        };
        // Issue order: S0_0 S1_0 | PV0_0 S0_1 | PV1_0 S1_1 | PV0_1 S0_2 | ...  While one
        // softmax group works on S_k, the tensor cores run the other group's P V and
        // its next S.  S_k(j+1) overwrites the columns PV_k(j) reads P_k(j) from; the
        // tcgen05.mma instructions of one thread execute in issue order.
        if (ok) ok = mbar_wait(bar_slot_full(slot_of(0)), 0, abort_flag, kSiteFwdMmaK);
        if (ok) {
          tc_fence_after();
          for (int k = 0; k < 2; ++k)
            if (act(k, 0)) issue_s(k, 0);
          mma_commit(bar_slot_empty(slot_of(0)));
        }
        for (int j = 0; j < n_kv && ok; ++j) {
          const int itV = 2 * j + 1, itK1 = 2 * j + 2;
          if (!(ok = mbar_wait(bar_slot_full(slot_of(itV)), (itV / C::NSLOT) & 1, abort_flag, kSiteFwdMmaV))) break;
          const bool more = j + 1 < n_kv;
          if (more &&
              !(ok = mbar_wait(bar_slot_full(slot_of(itK1)), (itK1 / C::NSLOT) & 1, abort_flag, kSiteFwdMmaK)))
            break;
          const uint32_t vaddr = sSlot0 + slot_of(itV) * C::TILE;
          for (int k = 0; k < 2; ++k) {
            if (!act(k, j)) continue;
            if (!(ok = mbar_wait(bar_p_full(k), j & 1, abort_flag, kSiteFwdMmaP))) break;
            tc_fence_after();
            const uint32_t tP = tmem + C::TM_S + k * 128;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)  // K = 128 keys, 16 per step = 8 TMEM columns of packed P
              mma_ts(tmem + C::TM_O + k * D, tP + kk * 8, sdesc_sw128(vaddr + kk * 2048, C::BLK), idPV,
                     (j > 0 || kk > 0) ? 1u : 0u);
            mma_commit(bar_pv_done(k));
            if (more && act(k, j + 1)) issue_s(k, j + 1);
          }
          if (!ok) break;
          mma_commit(bar_slot_empty(slot_of(itV)));
          if (more) mma_commit(bar_slot_empty(slot_of(itK1)));
        }
        // Make sure nothing this thread issued is still running before TMEM is freed.
        mma_commit(bar_drain);
        mbar_wait_ns(bar_drain, 0, 100000000ull);
      }
      __syncwarp();
    }
  } else {
    regs_increase<224>();
    // ------------------------------------------------------ softmax groups
    const int k = warp >> 2;  // query tile of this group
    const int wq = warp & 3;
    const int r = wq * 32 + lane;  // row inside the query tile
    const int n_kv_k = k == 0 ? n_kv0 : n_kv1;
    const int q_tile = tile0 + k;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tS = tmem + C::TM_S + k * 128 + lane_off;
    const uint32_t tO = tmem + C::TM_O + k * D + lane_off;
    const float sl2 = args.scale_log2;
    float m_ref = -INFINITY;  // reference max of the scaled scores, log2 units
    float l = 0.f;            // running sum of exp2(score - m_ref)
    bool ok = true;
    for (int j = 0; j < n_kv_k; ++j) {
      ok = mbar_wait(bar_s_full(k), j & 1, abort_flag, kSiteFwdSoftS);
      if (!(ok = __all_sync(0xffffffffu, ok))) break;
      tc_fence_after();
      uint32_t v[4][32];
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) tmem_ld32(tS + c4 * 32, v[c4]);
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) tmem_ld_wait(v[c4]);
      if (CAUSAL && j == q_tile) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c > r) v[c >> 5][c & 31] = __float_as_uint(sl2 >= 0.f ? -INFINITY : INFINITY);
      }
      // row max of the raw scores, turned into the max of scale * score (log2 units);
      // four independent three-input chains keep the dependencies short
      float mx;
      {
        float pm[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) pm[u] = __uint_as_float(v[u][0]);
        if (sl2 >= 0.f) {
#pragma unroll
          for (int c = 0; c < 128; c += 8)
#pragma unroll
            for (int u = 0; u < 4; ++u)
              pm[u] = fmax3(pm[u], __uint_as_float(v[(c + 2 * u) >> 5][(c + 2 * u) & 31]),
                            __uint_as_float(v[(c + 2 * u + 1) >> 5][(c + 2 * u + 1) & 31]));
          mx = fmax3(pm[0], pm[1], fmaxf(pm[2], pm[3]));
        } else {
#pragma unroll
          for (int c = 0; c < 128; c += 8)
#pragma unroll
            for (int u = 0; u < 4; ++u)
              pm[u] = fmin3(pm[u], __uint_as_float(v[(c + 2 * u) >> 5][(c + 2 * u) & 31]),
                            __uint_as_float(v[(c + 2 * u + 1) >> 5][(c + 2 * u + 1) & 31]));
          mx = fmin3(pm[0], pm[1], fminf(pm[2], pm[3]));
        }
        mx *= sl2;
      }
      // lazily move the reference max; rescale O and l only when it moves
      const bool grow = mx > m_ref + kRescaleThreshold;
      if (__any_sync(0xffffffffu, grow)) {
        const float m_new = fmaxf(m_ref, mx);
        const float alpha = ex2(m_ref - m_new);  // 0 on the first tile (m_ref = -inf)
        l *= alpha;
        m_ref = m_new;
        if (j > 0) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(tO + c * 32, o);
            tmem_ld_wait(o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(tO + c * 32, o);
          }
        }
      }
      const bool diag = CAUSAL && j == q_tile;  // keys c > r of this tile are masked
      const uint64_t sl2x2 = f2_pack(sl2, sl2), negm2 = f2_pack(-m_ref, -m_ref);
      uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};  // packed partial row sums
      uint32_t pk[2][32];                          // P row as packed bf16 pairs
#pragma unroll
      for (int c = 0; c < 128; c += 2) {
        const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(v[c >> 5][c & 31]),
                                           __uint_as_float(v[(c + 1) >> 5][(c + 1) & 31])),
                                   sl2x2, negm2);
        float p0, p1;
        if (((c >> 1) & 7) < kPolyPairsPer8) {
          f2_unpack(exp2_poly_x2(x2), p0, p1);  // on the FMA pipe
        } else {
          float x0, x1;
          f2_unpack(x2, x0, x1);
          p0 = ex2(x0);
          p1 = ex2(x1);
        }
        if (diag) {
          p0 = (c > r) ? 0.f : p0;
          p1 = (c + 1 > r) ? 0.f : p1;
        }
        acc[(c >> 1) & 3] = f2_add(acc[(c >> 1) & 3], f2_pack(p0, p1));
        pk[c >> 6][(c >> 1) & 31] = pack_bf16x2(p0, p1);
      }
      {
        const uint64_t a2 = f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3]));
        float s0, s1;
        f2_unpack(a2, s0, s1);
        l += s0 + s1;
      }
      // P (bf16 pairs) over the first 64 columns of S_k
      tmem_st32(tS, pk[0]);
      tmem_st32(tS + 32, pk[1]);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_p_full(k));
    }
    if (ok && n_kv_k > 0) {
      ok = __all_sync(0xffffffffu, mbar_wait(bar_pv_done(k), (n_kv_k - 1) & 1, abort_flag, kSiteFwdSoftO));
      if (ok) {
        tc_fence_after();
        const float inv_l = 1.f / l;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + c * 32, o);
          tmem_ld_wait(o);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const int chunk = (c & 1) * 4 + q4;
            const uint32_t* w = &o[q4 * 8];
            st_shared_v4(sQ(k) + (c >> 1) * C::BLK + sw128_offset(r, chunk),
                         pack_bf16x2(__uint_as_float(w[0]) * inv_l, __uint_as_float(w[1]) * inv_l),
                         pack_bf16x2(__uint_as_float(w[2]) * inv_l, __uint_as_float(w[3]) * inv_l),
                         pack_bf16x2(__uint_as_float(w[4]) * inv_l, __uint_as_float(w[5]) * inv_l),
                         pack_bf16x2(__uint_as_float(w[6]) * inv_l, __uint_as_float(w[7]) * inv_l));
          }
        }
        // natural-log LSE of the scaled scores: (m_ref + log2 l) * ln 2
        args.lse[head_row0 + q_tile * 128 + r] = (m_ref + __log2f(l)) * 0.69314718055994530942f;
        fence_async_shared();
        named_barrier(1 + k, 128);
        if (r == 0) {
#pragma unroll
          for (int kb = 0; kb < C::KB; ++kb)
            tma_store_2d(&tm_o, sQ(k) + kb * C::BLK, kb * 64, head_row0 + q_tile * 128);
          bulk_commit();
          bulk_wait0();
        }
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
