// dq_kernel.cuh -- the deterministic dQ pass of the exact-attention backward (sm_100a).
//
// The backward recomputes S and P tile by tile instead of reading a stored
// probability matrix (page 2 "四、反向传播选择重计算而非全量保存").  The default
// backward adds each key tile's dQ contribution into an fp32 accumulator with
// bulk reduce-adds (page 3 "5.3 专用指令利用": atomic global updates), whose order
// of fp32 additions varies from run to run.  This kernel instead owns one
// 128-row query tile and walks its key tiles in order, recomputing
//     S  = Q_i K_j^T,   P = exp2(S scale log2e - LSE2_i)   (masked),
//     dP = dO_i V_j^T,  dS = P o (dP o Z - D_i)
// and accumulating dQ_i += dS K_j in tensor memory, so every dQ element is one
// fixed sequence of operations: dQ is the same bit for bit on every run.  The
// dK/dV kernel then runs without its dQ product (fattn_bwd_dkdv_kernel with
// WITH_DQ = false).
//
// Roles (384 threads = three warpgroups):
//   warps 0..7  gradient warps.  Warpgroup h takes keys 64h .. 64h+63 of every
//               key tile; thread = query row of the tile.  Both write the dQ rows
//               at the end, warpgroup h the 32-column chunks c with c % 2 == h.
//   warp 8      TMA producer: Q_i, dO_i once; K_j, V_j through an NSLOT-deep ring
//   warp 9      tcgen05 issuer (the whole warp; lane 0 issues each instruction);
//               warps 10, 11 idle
// Tensor memory (512 columns): S in two buffers (columns 0 and 128; dS, bf16,
// overlays the first 32 columns of each 64-key half), dP at 256, dQ at 384.
// Issue order: S_0 dP_0 | S_1 dQ_0 dP_1 | S_2 dQ_1 dP_2 | ...: the exponentials of
// P_{j+1} overlap dQ_j and dP_{j+1}.
#pragma once

#include <type_traits>

#include "bwd_kernels.cuh"
#include "fwd_kernel.cuh"  // fwd_kv_tiles: the key tiles a query tile sees
#include "sm100.cuh"

namespace fattn {

struct DqArgs {
  const float* lse2;   // [B*H][stat_stride]  LSE * log2(e)
  const float* dvec;   // [B*H][stat_stride]  D
  __nv_bfloat16* dq;   // [B*H*N_q, D] bf16
  int N_q;
  int num_q_tiles;     // ceil(N_q / 128)
  int num_kv_tiles;    // ceil(N_k / 128)
  int stat_stride;     // num_q_tiles * 128
  int kv_tail;         // keys in the last key tile, 1..128
  int causal_off;      // N_k - N_q
  int G;               // query heads per key/value head
  int group_big;       // causal order: heads in each of the first num_big_groups groups;
  int num_big_groups;  //   the remaining groups hold group_big - 1 heads
  float scale;
  float scale_log2;
  sm100::Dropout drop;
};

template <int D>
struct DqCfg {
  using L = sm100::Cols<D>;
  static constexpr int TILE = 128 * D * 2;
  static constexpr int NSLOT = D == 128 ? 4 : D == 96 ? 4 : D == 64 ? 6 : 8;  // K/V ring
  static constexpr int OFF_Q = 0, OFF_DO = TILE, OFF_SLOT = 2 * TILE;
  static constexpr int OFF_BAR = OFF_SLOT + NSLOT * TILE;
  // q_full, slot_full[NSLOT], slot_empty[NSLOT], s_full[2], dp_full, ds_full, done, drain
  static constexpr int B_Q = 0, B_SF = 1, B_SE = 1 + NSLOT, B_S = 1 + 2 * NSLOT, B_DP = B_S + 2;
  static constexpr int B_DS = B_DP + 1, B_DONE = B_DP + 2, B_DRAIN = B_DP + 3;
  static constexpr int NBAR = B_DRAIN + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = OFF_MISC + 16;
  static_assert(SMEM <= 232448, "shared memory budget");
  static constexpr int TMEM_COLS = 512;
  static constexpr int TM_S = 0, TM_DP = 256, TM_DQ = 384;
};

enum : int {
  kSiteDqProducer = 0x301,
  kSiteDqMmaQ = 0x302,
  kSiteDqMmaK = 0x303,
  kSiteDqMmaV = 0x304,
  kSiteDqMmaDS = 0x305,
  kSiteDqSoftS = 0x306,
  kSiteDqSoftDP = 0x307,
  kSiteDqEpi = 0x308,
  kSiteDqAlign = 0x309,
};

template <int D, bool CAUSAL, bool DROPOUT>
__global__ void __launch_bounds__(384, 1)
    fattn_bwd_dq_pass_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                             const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                             const DqArgs args) {
  using C = DqCfg<D>;
  using namespace sm100;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_addr(smem);
  const uint32_t sQ = sbase + C::OFF_Q, sDO = sbase + C::OFF_DO, sSlot0 = sbase + C::OFF_SLOT;
  const uint32_t bar0 = sbase + C::OFF_BAR;
  auto bar = [&](int i) { return bar0 + 8u * i; };
  const uint32_t bar_q_full = bar(C::B_Q);
  auto bar_slot_full = [&](int s) { return bar(C::B_SF + s); };
  auto bar_slot_empty = [&](int s) { return bar(C::B_SE + s); };
  auto bar_s_full = [&](int b) { return bar(C::B_S + b); };
  const uint32_t bar_dp_full = bar(C::B_DP), bar_ds_full = bar(C::B_DS), bar_done = bar(C::B_DONE);
  const uint32_t bar_drain = bar(C::B_DRAIN);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (sbase & 1023u) {  // the swizzled layouts need 1024-byte alignment; never expected
    if (threadIdx.x == 0) atomicCAS(&g_fattn_status, 0, kSiteDqAlign);
    return;
  }
  const int NT = args.num_q_tiles, NKT = args.num_kv_tiles;
  // One CTA per (query head, query tile).  Causal: a query tile's work grows with
  // its index, so the heads form groups of group_big or group_big - 1 and inside
  // a group the longest tiles of all its heads come first.
  int bh, q_tile;
  if (CAUSAL) {
    const int big = args.group_big, ubig = NT * big, nbig_units = args.num_big_groups * ubig;
    const int u = (int)blockIdx.x;
    int r, hg, h0;
    if (u < nbig_units) {
      const int g = u / ubig;
      r = u - g * ubig;
      hg = big;
      h0 = g * big;
    } else {
      const int gs = NT * (big - 1), u2 = u - nbig_units, g = u2 / gs;
      r = u2 - g * gs;
      hg = big - 1;
      h0 = args.num_big_groups * big + g * (big - 1);
    }
    bh = h0 + r % hg;
    q_tile = NT - 1 - r / hg;
  } else {
    bh = (int)(blockIdx.x / (unsigned)NT);
    q_tile = (int)(blockIdx.x % (unsigned)NT);
  }
  const int kv_bh = bh / args.G;
  const int n_kv = fwd_kv_tiles(q_tile, NKT, args.causal_off, CAUSAL);

  if (threadIdx.x == 0) {
    mbar_init(bar_q_full, 1);
    for (int s = 0; s < C::NSLOT; ++s) {
      mbar_init(bar_slot_full(s), 1);
      mbar_init(bar_slot_empty(s), 1);
    }
    mbar_init(bar_s_full(0), 1);
    mbar_init(bar_s_full(1), 1);
    mbar_init(bar_dp_full, 1);
    mbar_init(bar_ds_full, 256);
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

  // 384 threads launch with 168 registers each (64512 in all): the producer/MMA
  // warpgroup keeps 56, the gradient warpgroups take 224 (2*128*224 + 128*56 = 64512).
  if (warp >= 8) {
    regs_decrease<56>();
    if (warp == 8) {
      // ---------------------------------------------------------- producer
      // The whole warp runs the loop and its waits; lane 0 alone issues the copies
      // and the barrier transactions (one()).
      {
        auto one = [&](auto f) { if (lane == 0) f(); __syncwarp(); };
        one([&] {
          prefetch_tensormap(&tm_q);
          prefetch_tensormap(&tm_k);
          prefetch_tensormap(&tm_v);
          prefetch_tensormap(&tm_do);
          mbar_arrive_expect_tx(bar_q_full, 2 * C::TILE);
#pragma unroll
          for (int kb = 0; kb < C::L::NB; ++kb) {
            tma_load_3d(sQ + kb * C::L::BLKB, &tm_q, bar_q_full, kb * C::L::CW, q_tile * 128, bh);
            tma_load_3d(sDO + kb * C::L::BLKB, &tm_do, bar_q_full, kb * C::L::CW, q_tile * 128, bh);
          }
        });
        int it = 0;  // tiles loaded: K_j at 2j, V_j at 2j + 1
        bool ok = true;
        for (int j = 0; j < n_kv && ok; ++j) {
          for (int t = 0; t < 2 && ok; ++t, ++it) {
            const int s = it % C::NSLOT;
            if (!(ok = mbar_wait(bar_slot_empty(s), ((it / C::NSLOT) & 1) ^ 1, abort_flag, kSiteDqProducer)))
              break;
            one([&] {
              mbar_arrive_expect_tx(bar_slot_full(s), C::TILE);
              const CUtensorMap* map = t == 0 ? &tm_k : &tm_v;
#pragma unroll
              for (int kb = 0; kb < C::L::NB; ++kb)
                tma_load_3d(sSlot0 + s * C::TILE + kb * C::L::BLKB, map, bar_slot_full(s), kb * C::L::CW, j * 128,
                            kv_bh);
            });
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
      // --------------------------------------------------------- MMA issuer
      // The whole warp runs this loop; lane 0 issues each tcgen05 instruction
      // (mma_*_warp).
      {
        constexpr uint32_t id_s = idesc_bf16_f32(128, 128, false, false);  // Q|dO (K-major) x K|V (K-major)
        constexpr uint32_t id_dq = idesc_bf16_f32(128, D, false, true);    // dS (TMEM) x K (MN-major)
        auto slot_addr = [&](int i) { return sSlot0 + (i % C::NSLOT) * C::TILE; };
        auto wait_slot = [&](int i, int site) {
          return mbar_wait(bar_slot_full(i % C::NSLOT), (i / C::NSLOT) & 1, abort_flag, site);
        };
        // dst = A B^T with K = D, both operands K-major 128-row tiles
        auto issue_rows = [&](uint32_t dst, uint32_t a_tile, uint32_t b_tile) {
          const uint64_t da = C::L::desc_k(opaque_u32(a_tile)), db = C::L::desc_k(opaque_u32(b_tile));
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off16 = C::L::kstep(kk) >> 4;
            mma_ss_warp(dst, da + off16, db + off16, id_s, kk > 0 ? 1u : 0u);
          }
        };
        bool ok = mbar_wait(bar_q_full, 0, abort_flag, kSiteDqMmaQ);
        if (ok) ok = wait_slot(0, kSiteDqMmaK);
        if (ok) {
          tc_fence_after();
          issue_rows(tmem + C::TM_S, sQ, slot_addr(0));  // S_0
          mma_commit_warp(bar_s_full(0));
          ok = wait_slot(1, kSiteDqMmaV);
        }
        if (ok) {
          tc_fence_after();
          issue_rows(tmem + C::TM_DP, sDO, slot_addr(1));  // dP_0
          mma_commit_warp(bar_dp_full);
        }
        for (int j = 0; j < n_kv && ok; ++j) {
          const int kslot = 2 * j, vslot = 2 * j + 1;
          if (j + 1 < n_kv) {
            // S_{j+1} into the other buffer: dQ_{j-1}, which read dS_{j-1} from
            // there, was issued before it, and one thread's tcgen05.mma execute in order
            if (!(ok = wait_slot(kslot + 2, kSiteDqMmaK))) break;
            tc_fence_after();
            issue_rows(tmem + C::TM_S + ((j + 1) & 1) * 128, sQ, slot_addr(kslot + 2));
            mma_commit_warp(bar_s_full((j + 1) & 1));
          }
          // dQ += dS_j K_j  (A = dS_j from TMEM, two 64-key halves; 8 steps of 16 keys)
          if (!(ok = mbar_wait(bar_ds_full, j & 1, abort_flag, kSiteDqMmaDS))) break;
          tc_fence_after();
          {
            const uint32_t tA = tmem + C::TM_S + (j & 1) * 128;
            const uint64_t db = C::L::desc_mn(opaque_u32(slot_addr(kslot)), C::L::BLKB);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)  // keys 16kk..: dS of half kk/4 at columns 64*(kk/4) + 8*(kk%4)
              mma_ts_warp(tmem + C::TM_DQ, tA + (kk >> 2) * 64 + (kk & 3) * 8, db + kk * (C::L::ROWSTEP16 >> 4), id_dq,
                     (j > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit_warp(bar_slot_empty(kslot % C::NSLOT));
          mma_commit_warp(bar_slot_empty(vslot % C::NSLOT));  // V_j's product dP_j was issued earlier
          if (j + 1 < n_kv) {
            // dP_{j+1}: the gradient warps read dP_j before they signalled dS_j
            if (!(ok = wait_slot(vslot + 2, kSiteDqMmaV))) break;
            tc_fence_after();
            issue_rows(tmem + C::TM_DP, sDO, slot_addr(vslot + 2));
            mma_commit_warp(bar_dp_full);
          }
        }
        if (ok) mma_commit_warp(bar_done);
        mma_commit_warp(bar_drain);
        mbar_wait_ns(bar_drain, 0, 100000000ull);
      }
      __syncwarp();
    }
  } else {
    regs_increase<224>();
    // ---------------------------------------------------------- gradient warps
    const int h = warp >> 2;       // key half: keys 64h .. 64h+63 of each tile
    const int wq = warp & 3;       // TMEM lane quarter of this warp
    const int r = wq * 32 + lane;  // query row of the tile
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const float sl2 = args.scale_log2;
    const size_t stat = (size_t)bh * args.stat_stride + q_tile * 128 + r;
    const float lse2_r = args.lse2[stat];
    const float d_r = args.dvec[stat];
    const uint32_t q_row = (uint32_t)(q_tile * 128 + r);
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const uint32_t tS = tmem + C::TM_S + (j & 1) * 128 + 64 * h + lane_off;
      ok = mbar_wait(bar_s_full(j & 1), (j >> 1) & 1, abort_flag, kSiteDqSoftS);
      if (!(ok = __all_sync(0xffffffffu, ok))) break;
      tc_fence_after();
      // Keys 64h + c < hi of this tile are visible: causal, key 128 j + 64 h + c is
      // visible to query 128 q_tile + r iff it is <= 128 q_tile + r + off; in a
      // ragged last tile the keys past N_k are not.
      int hi = 64;
      if (CAUSAL) hi = min(hi, 128 * (q_tile - j) + args.causal_off + 1 - 64 * h + r);
      if (j == NKT - 1) hi = min(hi, args.kv_tail - 64 * h);
      const bool any_mask = __any_sync(0xffffffffu, hi < 64);  // warp-uniform
      uint64_t keep = ~0ull;  // dropout keep bit of key 64h + c
      if constexpr (DROPOUT) {
        keep = 0;
        const uint32_t j4 = (uint32_t)(j * 128 + 64 * h) >> 2;
#pragma unroll
        for (int u = 0; u < 16; ++u)
          keep |= (uint64_t)dropout_keep4(args.drop, (uint32_t)bh, q_row, j4 + u) << (4 * u);
      }
      float p[64];
      {
        uint32_t v[2][32];
        tmem_ld32(tS, v[0]);
        tmem_ld32(tS + 32, v[1]);
        tmem_ld_wait(v[0]);
        tmem_ld_wait(v[1]);
        auto p_loop = [&](auto masked) {
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            const float e = ex2(fmaf(__uint_as_float(v[c >> 5][c & 31]), sl2, -lse2_r));
            if constexpr (decltype(masked)::value)
              p[c] = c < hi ? e : 0.f;
            else
              p[c] = e;
          }
        };
        if (any_mask)
          p_loop(std::true_type{});
        else
          p_loop(std::false_type{});
      }
      // dS = P o (dP o Z - D): dP for this half's keys, then dS as bf16 pairs over the
      // first 32 columns of this half's S (the A operand of dQ += dS K)
      ok = mbar_wait(bar_dp_full, j & 1, abort_flag, kSiteDqSoftDP);
      if (!(ok = __all_sync(0xffffffffu, ok))) break;
      tc_fence_after();
      uint32_t dsk[32];
#pragma unroll
      for (int c2 = 0; c2 < 2; ++c2) {
        uint32_t dv[32];
        tmem_ld32(tmem + C::TM_DP + 64 * h + c2 * 32 + lane_off, dv);
        tmem_ld_wait(dv);
#pragma unroll
        for (int t = 0; t < 32; t += 2) {
          const int c = c2 * 32 + t;
          float dp0 = __uint_as_float(dv[t]), dp1 = __uint_as_float(dv[t + 1]);
          if constexpr (DROPOUT) {
            dp0 = ((keep >> c) & 1ull) ? dp0 * args.drop.scale_keep : 0.f;
            dp1 = ((keep >> (c + 1)) & 1ull) ? dp1 * args.drop.scale_keep : 0.f;
          }
          dsk[c >> 1] = pack_bf16x2(p[c] * (dp0 - d_r), p[c + 1] * (dp1 - d_r));
        }
      }
      tmem_st32(tS, dsk);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_ds_full);
    }
    // dQ rows (thread = query row) -> scale -> bf16 -> global memory, 32 columns at a
    // time: warpgroup h takes the 32-column chunks c with c % 2 == h; rows past N_q
    // are not written
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_done, 0, abort_flag, kSiteDqEpi));
    if (ok) {
      tc_fence_after();
      const bool row_ok = q_tile * 128 + r < args.N_q;
      const float sc = args.scale;
      uint4* dst = reinterpret_cast<uint4*>(args.dq + ((size_t)bh * args.N_q + q_tile * 128 + r) * D);
#pragma unroll
      for (int c = h; c < D / 32; c += 2) {
        uint32_t o[32];
        tmem_ld32(tmem + C::TM_DQ + c * 32 + lane_off, o);
        tmem_ld_wait(o);
        if (row_ok) {
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const uint32_t* x = &o[q4 * 8];
            dst[c * 4 + q4] = make_uint4(pack_bf16x2(__uint_as_float(x[0]) * sc, __uint_as_float(x[1]) * sc),
                                         pack_bf16x2(__uint_as_float(x[2]) * sc, __uint_as_float(x[3]) * sc),
                                         pack_bf16x2(__uint_as_float(x[4]) * sc, __uint_as_float(x[5]) * sc),
                                         pack_bf16x2(__uint_as_float(x[6]) * sc, __uint_as_float(x[7]) * sc));
          }
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
