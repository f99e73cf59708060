// bwd_kernels.cuh -- exact-attention backward for sm_100a.
//
// The backward recomputes S and P tile by tile from Q, K and the saved
// log-sum-exp instead of reading a stored probability matrix (page 2 "四、反向
// 传播选择重计算而非全量保存").  Three kernels run in order on one stream:
//
//  1. fattn_bwd_pre_kernel   D_i = sum_c dO_ic O_ic, LSE2_i = LSE_i log2(e)
//                            (per head padded to whole 128-row tiles), and
//                            zero the fp32 dQ accumulator.         (HBM-bound)
//  2. fattn_bwd_dkdv_kernel  one CTA per (batch*head, 128-row key tile j);
//                            loops over the 128-row query tiles i that can see
//                            tile j and, on the tcgen05 tensor cores,
//                              S^T  = K_j Q_i^T          (TMEM)
//                              dP^T = V_j dO_i^T         (TMEM)
//                              P^T  = exp2(S^T scale log2e - LSE2_i)   (masked)
//                              dS^T = P^T o (dP^T - D_i)
//                              dV_j += P^T dO_i   (P^T read from TMEM)
//                              dK_j += dS^T Q_i   (dS^T read from TMEM)
//                              dQ_i^T = K_j^T dS^T_i -> staged in shared memory,
//                                  added into the fp32 accumulator by one TMA
//                                  bulk reduce per query tile
//                            (atomic global updates, page 3 "5.3 专用指令利用").
//                            A ragged last tile (N not a multiple of 128) is
//                            read as zeros past N through 3-D tensor maps; P
//                            is 0 for its queries and keys past N.
//  3. fattn_bwd_dq_kernel    dQ = bf16(scale * accumulator).
#pragma once

#include <type_traits>

#include "sm100.cuh"

namespace fattn {

// ------------------------------------------------------------------ kernel 1
template <int D>
__global__ void __launch_bounds__(256) fattn_bwd_pre_kernel(const __nv_bfloat16* __restrict__ o,
                                                            const __nv_bfloat16* __restrict__ dout,
                                                            const float* __restrict__ lse, float* __restrict__ dvec,
                                                            float* __restrict__ lse2, float* __restrict__ dq_acc,
                                                            long long heads, int N, int NP) {
  // One thread group per row of the padded statistics [heads][NP]: rows n < N get
  // D = sum(dO o O) and LSE * log2(e) and have their dQ accumulator row zeroed
  // (a row whose LSE is -inf -- no visible key -- has O = 0 and D = 0);
  // the padding rows of a ragged last tile get 0 (finite, and masked where used).
  // threads per row, 8-element (16-byte) pieces each: D / 8 of them for d = 64, 128;
  // 4 for d = 32, 96 (one and three pieces each), so that TPR is a power of two
  constexpr int TPR = D % 64 == 0 ? D / 8 : 4;
  constexpr int PIECES = D / (8 * TPR);
  constexpr int RPB = 256 / TPR;
  const long long prow = (long long)blockIdx.x * RPB + threadIdx.x / TPR;
  const bool in_range = prow < heads * NP;
  const long long bh = prow / NP;
  const int n = (int)(prow - bh * NP);
  const bool valid = in_range && n < N;
  const long long row = bh * N + n;
  const int part = threadIdx.x % TPR;
  float acc = 0.f;
  if (valid) {
#pragma unroll
    for (int pc = 0; pc < PIECES; ++pc) {
      const size_t off = (size_t)row * D + (part * PIECES + pc) * 8;
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
      if (dq_acc) {  // null for the deterministic backward, which has no accumulator
        float4* z = reinterpret_cast<float4*>(dq_acc + off);
        z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
        z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
  }
#pragma unroll
  for (int w = TPR / 2; w >= 1; w >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, w);
  if (in_range && part == 0) {
    dvec[prow] = valid ? acc : 0.f;
    lse2[prow] = valid ? lse[row] * 1.4426950408889634f : 0.f;
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
  const float* lse2;  // [B*H][stat_stride]  LSE * log2(e)
  const float* dvec;  // [B*H][stat_stride]  D
  float* dq_acc;      // [B*H*N_q, D] fp32 (unused without the dQ product)
  int N_q;
  int num_q_tiles;    // ceil(N_q / 128)
  int num_kv_tiles;   // ceil(N_k / 128)
  int stat_stride;    // num_q_tiles * 128: one head's padded statistics
  int q_tail;         // queries in the last 128-row query tile, 1..128
  int kv_tail;        // keys in the last 128-row key tile, 1..128
  int causal_off;     // N_k - N_q: query i sees keys j <= i + causal_off (causal)
  int G;              // query heads per key/value head (H / H_kv)
  int group_big;      // causal order: heads in each of the first num_big_groups groups;
  int num_big_groups; //   the remaining groups hold group_big - 1 heads
  float scale;        // for dK
  float scale_log2;   // scale * log2(e)
  sm100::Dropout drop;  // used by the DROPOUT instances only
};

// First query tile that sees key tile t (causal: query i sees key 128 t iff
// i >= 128 t - off); every key is seen by the last query, so it is < num_q_tiles.
__host__ __device__ inline int bwd_first_q_tile(int t, int off, bool causal) {
  if (!causal) return 0;
  const int first_row = 128 * t - off;
  return first_row <= 0 ? 0 : first_row / 128;
}

template <int D>
struct BwdCfg {
  using L = sm100::Cols<D>;                    // column blocks of a K, V, Q or dO tile
  static constexpr int NS = 2;                 // Q/dO ring depth
  static constexpr int TILE = 128 * D * 2;     // bytes of a 128-row K, V, Q or dO tile
  static constexpr int DS_BLK = 128 * 128;     // one 64-query block of dS^T (128-byte swizzle)
  static constexpr int DS_BYTES = 128 * 128 * 2;  // dS^T [128 keys][128 queries] bf16
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = TILE;
  static constexpr int OFF_STAGE = 2 * TILE;
  static constexpr int STAGE = 2 * TILE + 1024;  // Q tile, dO tile, LSE2[128], D[128]
  static constexpr int OFF_DS = OFF_STAGE + NS * STAGE;
  static constexpr int OFF_BAR = OFF_DS + DS_BYTES;
  // kv_full, q_full[NS], q_empty[NS], s_full, dp_full, p_full, ds_full, dq_full, dq_free, done, drain,
  // staged (dQ partial written to shared memory)
  // + staged1, qb_full[NS], qb_empty[NS]: the stage's dO half has barriers of its own
  static constexpr int NBAR = 1 + 2 * NS + 10 + 2 * NS;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = OFF_MISC + 16;  // the dynamic shared window starts 1024-byte aligned
  static constexpr int TMEM_COLS = 512;
  // Region A: S^T (fp32, column = query), then per 64-query half h: P^T (bf16
  // pairs) at columns 64h..64h+31 and dS^T at 64h+32..64h+63.
  // Region B: dP^T, then dQ^T.  Then the dV and dK accumulators.
  static constexpr int TM_A = 0, TM_B = 128, TM_DV = 256, TM_DK = 256 + D;
};

enum : int {
  kSiteBwdProducer = 0x201,
  kSiteBwdMmaKV = 0x202,
  kSiteBwdMmaQ = 0x203,
  kSiteBwdMmaP = 0x204,
  kSiteBwdMmaDS = 0x205,
  kSiteBwdMmaDQ = 0x206,
  kSiteBwdSoftS = 0x207,
  kSiteBwdSoftDP = 0x208,
  kSiteBwdDrain = 0x209,
  kSiteBwdEpi = 0x20a,
  kSiteBwdAlign = 0x20b,
};

// Roles (384 threads = three warpgroups):
//   warps 0..7   gradient warps.  Warpgroup h (warps 4h..4h+3) takes queries
//                64h..64h+63 of every query tile; thread = key row of the tile for
//                P^T and dS^T, thread = head-dim lane for its half of dQ^T.  Warps
//                4..7 also write dK and dV at the end.
//   warp 8       TMA producer (K, V once; Q/dO tiles through an NS-deep ring)
//   warp 9       tcgen05 issuer (the whole warp; lane 0 issues each instruction)
//   warp 10      dQ reducer (lane 0 issues): one bulk reduce-add per half of a query tile
//   warp 11      idle
// Per query tile i the tensor cores run
//   ... dV_i | dK_i dQ_i S_{i+1} | dP_{i+1} | dV_{i+1} | ...
// so that the exponentials of P_{i+1} (which need only S_{i+1}) overlap the dQ
// drain and dP_{i+1}, and dV_{i+1} overlaps the dS arithmetic.  Splitting each
// row's queries over two warpgroups halves the exponential and dS work on that
// chain.
template <int D, bool CAUSAL, bool DROPOUT, bool WITH_DQ>
__global__ void __launch_bounds__(384, 1)
    fattn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                          const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
                          const BwdArgs args) {
  using C = BwdCfg<D>;
  using namespace sm100;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_addr(smem);
  const uint32_t sK = sbase + C::OFF_K, sV = sbase + C::OFF_V, sDS = sbase + C::OFF_DS;
  auto sQ = [&](int s) { return sbase + C::OFF_STAGE + s * C::STAGE; };
  auto sDO = [&](int s) { return sbase + C::OFF_STAGE + s * C::STAGE + C::TILE; };
  auto sStat = [&](int s) { return sbase + C::OFF_STAGE + s * C::STAGE + 2 * C::TILE; };
  auto stat = [&](int s) { return reinterpret_cast<const float*>(smem + C::OFF_STAGE + s * C::STAGE + 2 * C::TILE); };
  const uint32_t bar0 = sbase + C::OFF_BAR;
  const uint32_t bar_kv_full = bar0;
  auto bar_q_full = [&](int s) { return bar0 + 8u * (1 + s); };
  auto bar_q_empty = [&](int s) { return bar0 + 8u * (1 + C::NS + s); };
  const uint32_t bar_s_full = bar0 + 8u * (1 + 2 * C::NS);
  const uint32_t bar_dp_full = bar_s_full + 8, bar_p_full = bar_s_full + 16, bar_ds_full = bar_s_full + 24;
  const uint32_t bar_dq_full = bar_s_full + 32, bar_dq_free = bar_s_full + 40, bar_done = bar_s_full + 48;
  const uint32_t bar_drain = bar_s_full + 56, bar_staged = bar_s_full + 64, bar_staged1 = bar_s_full + 72;
  // A Q/dO stage is two halves with their own full/empty barriers: Q and the
  // statistics (bar_q_full/bar_q_empty), and dO (bar_qb_full/bar_qb_empty).  The dQ^T
  // partial is staged with warpgroup 0's 64 queries over the Q half and warpgroup 1's
  // over the dO half, and each half goes back to the producer as soon as its own
  // bulk reduce has read it, so that Q_{i+2} (needed first, for S) loads early.
  auto bar_qb_full = [&](int s) { return bar0 + 8u * (1 + 2 * C::NS + 10 + s); };
  auto bar_qb_empty = [&](int s) { return bar0 + 8u * (1 + 2 * C::NS + 10 + C::NS + s); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (sbase & 1023u) {  // the swizzled layouts need 1024-byte alignment; never expected
    if (threadIdx.x == 0) atomicCAS(&g_fattn_status, 0, kSiteBwdAlign);
    return;
  }
  const int NT = args.num_q_tiles;
  const int NKT = args.num_kv_tiles;
  // One CTA per (key/value head, key tile).  Non-causal: the key tile varies
  // fastest, so the CTAs resident at one time add into the same heads' dQ rows
  // (which then stay in L2).  Causal: a key tile's work falls with its index, so
  // the heads form groups of group_big or group_big - 1 and inside a group the
  // longest tiles of all its heads come first; CTAs start in block order as SMs
  // free up, which makes this longest-first list scheduling within an L2-sized
  // set of heads.
  int bh, kv_tile;  // bh: flattened key/value head b * H_kv + hk
  if (CAUSAL) {
    const int big = args.group_big, ubig = NKT * big, nbig_units = args.num_big_groups * ubig;
    const int u = (int)blockIdx.x;
    int r, hg, h0;
    if (u < nbig_units) {
      const int g = u / ubig;
      r = u - g * ubig;
      hg = big;
      h0 = g * big;
    } else {
      const int gs = NKT * (big - 1), u2 = u - nbig_units, g = u2 / gs;
      r = u2 - g * gs;
      hg = big - 1;
      h0 = args.num_big_groups * big + g * (big - 1);
    }
    bh = h0 + r % hg;
    kv_tile = r / hg;
  } else {
    bh = (int)(blockIdx.x / (unsigned)NKT);
    kv_tile = (int)(blockIdx.x % (unsigned)NKT);
  }
  // Steps: the G query heads that share this key/value head, one after the other,
  // each over its query tiles i_begin .. NT - 1 (those that see this key tile).
  const int i_begin = bwd_first_q_tile(kv_tile, args.causal_off, CAUSAL);
  const int n_head = NT - i_begin;
  const int n_it = args.G * n_head;
  // step it = g * n_head + qi: query head bh * G + g (= b*H + h), query tile i_begin + qi,
  // kept as running counters (no division per step)
  struct Step {
    int g = 0, qi = 0;
    __device__ void next(int n) {
      if (++qi == n) {
        qi = 0;
        ++g;
      }
    }
  };

  if (threadIdx.x == 0) {
    mbar_init(bar_kv_full, 1);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(bar_q_full(s), 1);
      mbar_init(bar_q_empty(s), 1);
      mbar_init(bar_qb_full(s), 1);
      mbar_init(bar_qb_empty(s), 1);
    }
    mbar_init(bar_s_full, 1);
    mbar_init(bar_dp_full, 1);
    mbar_init(bar_p_full, 256);
    mbar_init(bar_ds_full, 256);
    mbar_init(bar_dq_full, 1);
    mbar_init(bar_dq_free, 256);
    mbar_init(bar_done, 1);
    mbar_init(bar_drain, 1);
    mbar_init(bar_staged, 128);
    mbar_init(bar_staged1, 128);
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

  // 384 threads launch with 168 registers each (64512 in all): the producer/MMA
  // warpgroup keeps 88, the other two take 208 (2*128*208 + 128*88 = 64512); with
  // 56 for the producer/MMA group its loop state spilled.
  if (warp >= 8) {
    regs_decrease<88>();
    if (warp == 8) {
      // ---------------------------------------------------------- producer
      // The whole warp runs the loop and its waits; lane 0 alone issues the copies
      // and the barrier transactions (one()).  A lone lane running the loop competes
      // for issue slots with the gradient warps beside it.
      {
        auto one = [&](auto f) { if (lane == 0) f(); __syncwarp(); };
        one([&] {
          prefetch_tensormap(&tm_q);
          prefetch_tensormap(&tm_k);
          prefetch_tensormap(&tm_v);
          prefetch_tensormap(&tm_do);
          mbar_arrive_expect_tx(bar_kv_full, 2 * C::TILE);
#pragma unroll
          for (int kb = 0; kb < C::L::NB; ++kb) {
            tma_load_3d(sK + kb * C::L::BLKB, &tm_k, bar_kv_full, kb * C::L::CW, kv_tile * 128, bh);
            tma_load_3d(sV + kb * C::L::BLKB, &tm_v, bar_kv_full, kb * C::L::CW, kv_tile * 128, bh);
          }
        });
        int it = 0;
        int half_issued = 0;  // stage halves whose loads went out (2 per step)
        Step sx;
        for (; it < n_it; ++it, sx.next(n_head)) {
          const int s = it % C::NS;
          if (!mbar_wait(bar_q_empty(s), ((it / C::NS) & 1) ^ 1, abort_flag, kSiteBwdProducer)) break;
          const int q_tile = i_begin + sx.qi, qh = bh * args.G + sx.g;
          const size_t stat_row = (size_t)qh * args.stat_stride + q_tile * 128;
          one([&] {
            mbar_arrive_expect_tx(bar_q_full(s), C::TILE + 1024);
#pragma unroll
            for (int kb = 0; kb < C::L::NB; ++kb)
              tma_load_3d(sQ(s) + kb * C::L::BLKB, &tm_q, bar_q_full(s), kb * C::L::CW, q_tile * 128, qh);
            bulk_load(sStat(s), args.lse2 + stat_row, 512, bar_q_full(s));
            bulk_load(sStat(s) + 512, args.dvec + stat_row, 512, bar_q_full(s));
          });
          ++half_issued;
          if (!mbar_wait(bar_qb_empty(s), ((it / C::NS) & 1) ^ 1, abort_flag, kSiteBwdProducer)) break;
          one([&] {
            mbar_arrive_expect_tx(bar_qb_full(s), C::TILE);
#pragma unroll
            for (int kb = 0; kb < C::L::NB; ++kb)
              tma_load_3d(sDO(s) + kb * C::L::BLKB, &tm_do, bar_qb_full(s), kb * C::L::CW, q_tile * 128, qh);
          });
          ++half_issued;
        }
        if (it < n_it) {  // aborted: let the copies already issued land
          mbar_wait_ns(bar_kv_full, 0, 100000000ull);
          for (int i = (it > C::NS ? it - C::NS : 0); i <= it && i < n_it; ++i) {
            if (2 * i < half_issued) mbar_wait_ns(bar_q_full(i % C::NS), (i / C::NS) & 1, 100000000ull);
            if (2 * i + 1 < half_issued) mbar_wait_ns(bar_qb_full(i % C::NS), (i / C::NS) & 1, 100000000ull);
          }
        }
      }
      __syncwarp();
    } else if (warp == 9) {
      // --------------------------------------------------------- MMA issuer
      // The whole warp runs this loop; lane 0 issues each tcgen05 instruction
      // (mma_*_warp).
      {
        constexpr uint32_t id_s = idesc_bf16_f32(128, 128, false, false);  // K|V (K-major) x Q|dO (K-major)
        constexpr uint32_t id_kv = idesc_bf16_f32(128, D, false, true);    // P^T|dS^T (TMEM) x dO|Q (MN)
        constexpr uint32_t id_q = idesc_bf16_f32(128, 128, true, true);    // K^T (MN) x dS^T (MN)
        // For d = 64 the dQ^T product still uses M = 128: the second 64-row half of
        // A repeats the first (LBO = 0) and its output lanes are ignored.
        // (d = 32 likewise repeats its one block four times; for d = 96 the fourth
        // block lies past K, inside the V tile, and only feeds the ignored lanes 96..127)
        constexpr uint32_t kt_lbo = C::L::NB > 1 ? C::L::BLKB : 0;
        const uint32_t tA = tmem + C::TM_A, tB = tmem + C::TM_B;
        // Descriptors: the start address is a descriptor's low 14 bits (address /
        // 16, below 2^14 for any shared-memory address), so each K step adds a
        // constant to one base descriptor per operand.  The base addresses pass
        // through an opaque move, so that the descriptors of every tile and step
        // are not hoisted out of the loop into this thread's 56 registers.
        auto issue_kxq = [&](uint32_t dst, uint32_t a_tile, uint32_t b_tile) {  // dst = A_tile B_tile^T, K = D
          const uint64_t da = C::L::desc_k(opaque_u32(a_tile)), db = C::L::desc_k(opaque_u32(b_tile));
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off16 = C::L::kstep(kk) >> 4;
            mma_ss_warp(dst, da + off16, db + off16, id_s, kk > 0 ? 1u : 0u);
          }
        };
        bool ok = mbar_wait(bar_kv_full, 0, abort_flag, kSiteBwdMmaKV);
        if (ok) ok = mbar_wait(bar_q_full(0), 0, abort_flag, kSiteBwdMmaQ);
        if (ok) {
          tc_fence_after();
          issue_kxq(tA, sK, sQ(0));  // S^T_0
          mma_commit_warp(bar_s_full);
          ok = mbar_wait(bar_qb_full(0), 0, abort_flag, kSiteBwdMmaQ);
        }
        if (ok) {
          tc_fence_after();
          issue_kxq(tB, sV, sDO(0));  // dP^T_0
          mma_commit_warp(bar_dp_full);
        }
        for (int it = 0; it < n_it && ok; ++it) {
          const int s = it % C::NS;
          // dV += P^T dO  (A = P^T from TMEM, two 64-query halves; 8 steps of 16 queries)
          if (!(ok = mbar_wait(bar_p_full, it & 1, abort_flag, kSiteBwdMmaP))) break;
          tc_fence_after();
          {
            const uint64_t db = C::L::desc_mn(opaque_u32(sDO(s)), C::L::BLKB);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)  // queries 16kk..: P^T of half kk/4 at columns 64*(kk/4) + 8*(kk%4)
              mma_ts_warp(tmem + C::TM_DV, tA + (kk >> 2) * 64 + (kk & 3) * 8, db + kk * (C::L::ROWSTEP16 >> 4), id_kv,
                     (it > 0 || kk > 0) ? 1u : 0u);
          }
          // dK += dS^T Q  (A = dS^T from TMEM, two 64-query halves)
          if (!(ok = mbar_wait(bar_ds_full, it & 1, abort_flag, kSiteBwdMmaDS))) break;
          tc_fence_after();
          {
            const uint64_t db = C::L::desc_mn(opaque_u32(sQ(s)), C::L::BLKB);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)  // dS^T of half kk/4 at columns 64*(kk/4) + 32 + 8*(kk%4)
              mma_ts_warp(tmem + C::TM_DK, tA + (kk >> 2) * 64 + 32 + (kk & 3) * 8, db + kk * (C::L::ROWSTEP16 >> 4),
                     id_kv,
                     (it > 0 || kk > 0) ? 1u : 0u);
          }
          if constexpr (WITH_DQ) {
            // (the Q/dO stage is released by the dQ drain, which reuses it as staging)
            // dQ^T = K^T dS^T into region B (dP^T already read)
            const uint64_t da = C::L::desc_mn(opaque_u32(sK), kt_lbo), db = sdesc_sw128(opaque_u32(sDS), C::DS_BLK);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)  // 16 keys per step: 16 rows of K, 16 rows of dS^T
              mma_ss_warp(tB, da + kk * (C::L::ROWSTEP16 >> 4), db + kk * (2048 >> 4), id_q, kk > 0 ? 1u : 0u);
            mma_commit_warp(bar_dq_full);
          } else {
            mma_commit_warp(bar_q_empty(s));  // dV_i and dK_i were the stage's last readers
            mma_commit_warp(bar_qb_empty(s));
          }
          if (it + 1 < n_it) {
            const int s1 = (it + 1) % C::NS;
            if (!(ok = mbar_wait(bar_q_full(s1), ((it + 1) / C::NS) & 1, abort_flag, kSiteBwdMmaQ))) break;
            tc_fence_after();
            // S^T_{i+1} over region A: the dV/dK products reading P^T/dS^T were
            // issued before it, and tcgen05.mma of one thread executes in order
            issue_kxq(tA, sK, sQ(s1));
            mma_commit_warp(bar_s_full);
            // dP^T_{i+1} over region B once dQ^T_i has been drained (without the dQ
            // product, once dP^T_i was read: the gradient warps did so before ds_full)
            if constexpr (WITH_DQ) {
              if (!(ok = mbar_wait(bar_dq_free, it & 1, abort_flag, kSiteBwdMmaDQ))) break;
            }
            if (!(ok = mbar_wait(bar_qb_full(s1), ((it + 1) / C::NS) & 1, abort_flag, kSiteBwdMmaQ))) break;
            tc_fence_after();
            issue_kxq(tB, sV, sDO(s1));
            mma_commit_warp(bar_dp_full);
          }
        }
        if (ok) mma_commit_warp(bar_done);
        mma_commit_warp(bar_drain);
        mbar_wait_ns(bar_drain, 0, 100000000ull);
      }
      __syncwarp();
    } else if (warp == 10) {
      // ---------------------------------------------------------- dQ reducer
      // The gradient warps stage dQ^T_i as row-major fp32 [128 queries][D] in step
      // i's Q/dO stage; one TMA bulk reduce-add puts it into the accumulator rows,
      // which are contiguous.  The stage goes back to the producer once the reduce
      // has read it, without holding up a gradient warp meanwhile.
      // As in the producer, the whole warp runs the loop, lane 0 issues (one()).
      if (WITH_DQ) {
        auto one = [&](auto f) { if (lane == 0) f(); __syncwarp(); };
        Step sx;
        for (int it = 0; it < n_it; ++it, sx.next(n_head)) {
          const int s = it % C::NS;
          // only the tile's rows inside the sequence (a ragged last tile has fewer)
          const int q_tile = i_begin + sx.qi;
          const int rows = q_tile == NT - 1 ? args.q_tail : 128;
          const int rows0 = rows < 64 ? rows : 64, rows1 = rows - rows0;
          float* dst = args.dq_acc + ((size_t)(bh * args.G + sx.g) * args.N_q + q_tile * 128) * D;
          // queries 0..63 (warpgroup 0), staged over the Q half; then 64..127 over the dO half
          if (!mbar_wait(bar_staged, it & 1, abort_flag, kSiteBwdDrain)) break;
          one([&] {
            bulk_reduce_add_f32(dst, sQ(s), (uint32_t)(rows0 * D * 4));
            bulk_commit();
            bulk_wait_read0();
            mbar_arrive(bar_q_empty(s));  // the producer may load the next Q here
          });
          if (!mbar_wait(bar_staged1, it & 1, abort_flag, kSiteBwdDrain)) break;
          one([&] {
            if (rows1 > 0) {
              bulk_reduce_add_f32(dst + 64 * D, sDO(s), (uint32_t)(rows1 * D * 4));
              bulk_commit();
              bulk_wait_read0();
            }
            mbar_arrive(bar_qb_empty(s));  // ... and the next dO here
          });
        }
        one([&] { bulk_wait0(); });  // the last reduce has landed in global memory
      }
      __syncwarp();
    }
  } else {
    regs_increase<208>();
    // ---------------------------------------------------------- gradient warps
    const int h = warp >> 2;   // query half: queries 64h .. 64h+63 of each tile
    const int wq = warp & 3;   // TMEM lane quarter of this warp
    const int r = wq * 32 + lane;  // key row (P^T, dS^T), head-dim lane (dQ^T)
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tA = tmem + C::TM_A + lane_off, tB = tmem + C::TM_B + lane_off;
    const float sl2 = args.scale_log2;
    const bool has_d = r < D;  // TMEM lane = head-dim index of dQ^T
    bool ok = true;
    Step sx;
    for (int it = 0; it < n_it; ++it, sx.next(n_head)) {
      const int s = it % C::NS;
      ok = mbar_wait(bar_s_full, it & 1, abort_flag, kSiteBwdSoftS);
      ok = ok && mbar_wait(bar_q_full(s), (it / C::NS) & 1, abort_flag, kSiteBwdSoftS);
      if (!(ok = __all_sync(0xffffffffu, ok))) break;
      tc_fence_after();
      const float* lse_s = stat(s) + 64 * h;
      const float* dvec_s = stat(s) + 128 + 64 * h;
      const int q_tile = i_begin + sx.qi;
      // P = 0 outside the window lo <= c < hi of this half's 64 queries.  Causal:
      // query 128 q_tile + 64 h + c sees key 128 kv_tile + r iff c >= lo, lo =
      // 128 (kv_tile - q_tile) - off - 64 h + r (> 0 only near the diagonal).  In a
      // ragged last query tile the queries past the sequence, and for a key past
      // the sequence every query, are outside too.
      const int q_valid = q_tile == NT - 1 ? args.q_tail - 64 * h : 64;
      const bool k_out = kv_tile == NKT - 1 && r >= args.kv_tail;
      const int lo = CAUSAL ? 128 * (kv_tile - q_tile) - args.causal_off - 64 * h + r : 0;
      const int hi = k_out ? 0 : q_valid;
      // Dropout: bit c of keep = keep bit of (query 128 q_tile + 64 h + c, this key).
      // One generator call gives four consecutive keys of one query -- the keys of
      // the four lanes of a quad -- so each lane of a quad draws every fourth query
      // (16 calls) and the quad swaps the bits with four shuffles.
      uint64_t keep = ~0ull;
      if constexpr (DROPOUT) {
        const int m = lane & 3;
        const uint32_t j4 = (uint32_t)(kv_tile * 128 + r) >> 2;  // the same for the whole quad
        const uint32_t i0 = (uint32_t)(q_tile * 128 + 64 * h);
        const uint32_t qh = (uint32_t)(bh * args.G + sx.g);
        uint64_t mine = 0;  // bits 4t .. 4t+3: keys of the quad, query i0 + 4t + m
#pragma unroll
        for (int t = 0; t < 16; ++t)
          mine |= (uint64_t)dropout_keep4(args.drop, qh, i0 + 4 * t + m, j4) << (4 * t);
        keep = 0;
#pragma unroll
        for (int src = 0; src < 4; ++src) {  // queries i0 + 4t + src come from quad lane src
          const uint64_t x = __shfl_sync(0xffffffffu, mine, (lane & ~3) | src) >> m;
#pragma unroll
          for (int t = 0; t < 16; ++t) keep |= ((x >> (4 * t)) & 1ull) << (4 * t + src);
        }
      }
      auto zf = [&](int c) { return ((keep >> c) & 1ull) ? args.drop.scale_keep : 0.f; };
      const bool any_mask = __any_sync(0xffffffffu, lo > 0 || hi < 64);  // warp-uniform
      // P^T row, this warpgroup's 64 queries: kept in fp32 for dS, packed to bf16 for dV
      float p[64];
      {
        uint32_t v[2][32];
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) tmem_ld32(tA + 64 * h + c2 * 32, v[c2]);
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) tmem_ld_wait(v[c2]);
        auto p_loop = [&](auto masked) {
#pragma unroll
          for (int c = 0; c < 64; c += 4) {
            const float4 l4 = *reinterpret_cast<const float4*>(lse_s + c);  // one broadcast load per 4 columns
            const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
            float e[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
              e[u] = ex2(fmaf(__uint_as_float(v[(c + u) >> 5][(c + u) & 31]), sl2, -lv[u]));
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              if constexpr (decltype(masked)::value)
                p[c + u] = (c + u < lo || c + u >= hi) ? 0.f : e[u];
              else
                p[c + u] = e[u];
            }
          }
        };
        if (any_mask)
          p_loop(std::true_type{});
        else
          p_loop(std::false_type{});
      }
      {
        uint32_t pk[32];
        if constexpr (DROPOUT) {  // dV takes the dropped, rescaled weights
#pragma unroll
          for (int c = 0; c < 64; c += 2) pk[c >> 1] = pack_bf16x2(p[c] * zf(c), p[c + 1] * zf(c + 1));
        } else {
#pragma unroll
          for (int c = 0; c < 64; c += 2) pk[c >> 1] = pack_bf16x2(p[c], p[c + 1]);
        }
        // bf16 pairs into columns 64h .. 64h+31: inside this warpgroup's own S^T
        // columns, which the other warpgroup never reads
        tmem_st32(tA + 64 * h, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_p_full);
      // dS^T = P^T o (dP^T - D), 32 queries at a time
      ok = mbar_wait(bar_dp_full, it & 1, abort_flag, kSiteBwdSoftDP);
      if (!(ok = __all_sync(0xffffffffu, ok))) break;
      tc_fence_after();
#pragma unroll
      for (int c2 = 0; c2 < 2; ++c2) {
        uint32_t dv[32];
        tmem_ld32(tB + 64 * h + c2 * 32, dv);
        tmem_ld_wait(dv);
        if constexpr (DROPOUT) {  // dP = (dO V^T) o Z
#pragma unroll
          for (int t = 0; t < 32; ++t) dv[t] = __float_as_uint(__uint_as_float(dv[t]) * zf(c2 * 32 + t));
        }
        uint32_t dsk[16];
#pragma unroll
        for (int t = 0; t < 16; t += 2) {
          const int c = c2 * 32 + 2 * t;
          const float4 d4 = *reinterpret_cast<const float4*>(dvec_s + c);  // one broadcast load per 4 columns
          dsk[t] = pack_bf16x2(p[c] * (__uint_as_float(dv[2 * t]) - d4.x),
                               p[c + 1] * (__uint_as_float(dv[2 * t + 1]) - d4.y));
          dsk[t + 1] = pack_bf16x2(p[c + 2] * (__uint_as_float(dv[2 * t + 2]) - d4.z),
                                   p[c + 3] * (__uint_as_float(dv[2 * t + 3]) - d4.w));
        }
        tmem_st16(tA + 64 * h + 32 + c2 * 16, dsk);  // columns 64h+32 .. 64h+63
        if constexpr (WITH_DQ) {
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4)  // 16-byte chunk c2*4+q4 of the 64-query block h
            st_shared_v4(sDS + h * C::DS_BLK + sw128_offset(r, c2 * 4 + q4), dsk[q4 * 4], dsk[q4 * 4 + 1],
                         dsk[q4 * 4 + 2], dsk[q4 * 4 + 3]);
        }
      }
      tmem_st_wait();
      if constexpr (WITH_DQ) fence_async_shared();
      tc_fence_before();
      mbar_arrive(bar_ds_full);
      if constexpr (!WITH_DQ) continue;
      // dQ^T_i, this warpgroup's 64 queries -> shared memory as row-major fp32
      // [128 queries][D] in this step's Q/dO stage (free: its last readers, dV_i and
      // dK_i, completed before dQ^T_i) for the reducer's bulk reduce-add
      ok = mbar_wait(bar_dq_full, it & 1, abort_flag, kSiteBwdDrain);
      if (!(ok = __all_sync(0xffffffffu, ok))) break;
      tc_fence_after();
      uint32_t v[2][32];
      if (has_d) {
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) tmem_ld32(tB + 64 * h + c2 * 32, v[c2]);
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) tmem_ld_wait(v[c2]);
      }
      tc_fence_before();
      mbar_arrive(bar_dq_free);
      if (has_d) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          st_shared_f32(sQ(s) + (uint32_t)((64 * h + c) * D + r) * 4u, __uint_as_float(v[c >> 5][c & 31]));
      }
      fence_async_shared();
      mbar_arrive(h == 0 ? bar_staged : bar_staged1);
    }
    if (h == 1) {
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_done, 0, abort_flag, kSiteBwdEpi));
      if (ok) {
        tc_fence_after();
        // dV, dK rows (thread = key row) -> bf16 -> the now idle V and K tiles -> TMA store
        const int row = r;
#pragma unroll
        for (int which = 0; which < 2; ++which) {
          const uint32_t tsrc = tmem + (which ? C::TM_DK : C::TM_DV) + lane_off;
          const uint32_t sdst = which ? sK : sV;
          const float mul = which ? args.scale : 1.f;
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t w32[32];
            tmem_ld32(tsrc + c * 32, w32);
            tmem_ld_wait(w32);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {  // columns c*32 + 8 q4 .. +7: block, then 16-byte chunk in it
              const int col = c * 32 + q4 * 8;
              const uint32_t* w = &w32[q4 * 8];
              st_shared_v4(sdst + (col / C::L::CW) * C::L::BLKB + C::L::chunk_offset(row, (col % C::L::CW) / 8),
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
          for (int kb = 0; kb < C::L::NB; ++kb) {
            // 3-D stores: rows of a ragged last key tile past the sequence are not written
            tma_store_3d(&tm_dv, sV + kb * C::L::BLKB, kb * C::L::CW, kv_tile * 128, bh);
            tma_store_3d(&tm_dk, sK + kb * C::L::BLKB, kb * C::L::CW, kv_tile * 128, bh);
          }
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
