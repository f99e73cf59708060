// fwd_kernel.cuh -- fused exact-attention forward for sm_100a.
//
// A persistent CTA (one per SM) loops over work units, each two consecutive
// 128-row query tiles of one (batch, head).  It streams the 128-row key/value
// tiles of that head through a shared-memory ring and keeps the running row max
// m and row sum l of the online softmax in registers, so the N x N score matrix
// never leaves the chip (page 2 "一、用分块
// 计算提高片上数据复用" and "二、在线 Softmax 保持精确结果"; page 3 "4.1 分块计算"
// and "4.2 在线softmax技巧").  Only O and the per-row log-sum-exp are written
// (page 2 "三、融合算子减少中间张量落盘").
//
// Roles (384 threads = three warpgroups, warp-specialised):
//   warps 0..3  softmax group 0, thread = row of query tile 0   (208 registers)
//   warps 4..7  softmax group 1, thread = row of query tile 1   (208 registers)
//   warp 8      TMA producer: Q tiles through a 3-buffer ring, K_j, V_j through
//               an NSLOT-deep ring; it also hands the work units to the others
//   warp 9      tcgen05 issuer (the whole warp; lane 0 issues each instruction);
//               warps 10, 11 idle                                 (88 registers)
//                 S0 = Q0 K_j^T, S1 = Q1 K_j^T          (TMEM, fp32)
//                 O0 += P0 V_j,  O1 += P1 V_j           (P read from TMEM)
// While group 0 turns S0 into P0 the tensor cores compute S1 (and vice versa),
// so the exponentials of one tile overlap the products of the other.  The Q
// ring has a third buffer, so the next unit's first query tile loads while the
// current unit still holds two.
//
// Tensor memory (512 columns x 128 lanes): S0 at column 0, S1 at 128 (P_k, bf16,
// overlays the first 64 columns of S_k), O0 at 256, O1 at 256 + D.
//
// Any N: the tiles stay 128 rows, and the 3-D tensor maps read a ragged last
// tile's rows past N as zero.  Its keys past N are masked (non-causal; the causal
// mask already hides them from every query before N), and its rows past N are
// not stored.
//
// Online softmax with a lazily updated reference max: each row keeps a
// reference m_ref (log2 units) and sums exp2(s - m_ref).  When a tile's row max
// exceeds m_ref by more than kRescaleThreshold, m_ref moves up and the partial
// O and l are multiplied by exp2(m_old - m_new) (page 2: "按照新的数值尺度修正此
// 前的累加结果").  Otherwise m_ref stays, weights stay <= 2^threshold, and since O
// and l share the same reference the final O / l is unchanged.
#pragma once

#include <type_traits>

#include "sm100.cuh"

namespace fattn {

struct FwdArgs {
  float* lse;            // [B*H*N_q] fp32
  __nv_bfloat16* o;      // [B*H*N_q, D] bf16
  int N_q;               // queries per head
  int num_q_tiles;       // ceil(N_q / 128)
  int num_kv_tiles;      // ceil(N_k / 128)
  int kv_tail;           // keys in the last 128-key tile, 1..128
  int causal_off;        // N_k - N_q: query i sees keys j <= i + causal_off (causal)
  int G;                 // query heads per key/value head (H / H_kv)
  int num_units;         // B*H * ceil(num_q_tiles / 2)
  int group_big;         // causal order: heads in each of the first num_big_groups groups;
  int num_big_groups;    //   the remaining groups hold group_big - 1 heads
  // Causal only, may be null: two device counters (next unit ticket, CTAs
  // finished), both 0 at launch and returned to 0 by the last CTA.  With them
  // each CTA claims its next unit when it runs short of work; without them CTA c
  // takes units c, c + gridDim.x, ...
  unsigned int* sched;
  float scale_log2;      // scale * log2(e)
  sm100::Dropout drop;   // used by the DROPOUT instances only
};

// Key tiles query tile t needs (from tile 0 on): all of them, or, causal, those up to
// the one holding key 128 t + 127 + off; at least 1 (a tile whose rows see no key
// still runs once, fully masked, so that its O = 0 and LSE = -inf are written).
__host__ __device__ inline int fwd_kv_tiles(int t, int nkt, int off, bool causal) {
  if (!causal) return nkt;
  const int last = 128 * t + 127 + off;  // last key any row of the tile sees
  if (last < 0) return 1;
  const int n = last / 128 + 1;
  return n < nkt ? n : nkt;
}

template <int D>
struct FwdCfg {
  using L = sm100::Cols<D>;                         // column blocks of a tile
  static constexpr int TILE = 128 * D * 2;          // bytes of one 128-row Q/K/V tile
  static constexpr int QBUF = 3;                    // Q tile ring
  static constexpr int NSLOT = D == 128 ? 4 : D == 96 ? 6 : D == 64 ? 6 : 8;  // K/V ring depth
  static constexpr int NUNIT = 4;                   // ring of unit indices from the producer
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_SLOT = QBUF * TILE;
  static constexpr int OFF_BAR = OFF_SLOT + NSLOT * TILE;
  // barriers: q_full[QBUF], q_empty[QBUF], slot_full[NSLOT], slot_empty[NSLOT],
  // s_full[2], p_full[2], pv_done[2], o_free[2], drain, unit_full[NUNIT], unit_empty[NUNIT]
  static constexpr int B_QF = 0, B_QE = QBUF, B_SF = 2 * QBUF, B_SE = B_SF + NSLOT;
  static constexpr int B_S = B_SE + NSLOT, B_P = B_S + 2, B_PV = B_S + 4, B_OF = B_S + 6;
  static constexpr int B_DRAIN = B_S + 8, B_UF = B_DRAIN + 1, B_UE = B_UF + NUNIT;
  static constexpr int NBAR = B_UE + NUNIT;
  // tmem base (4 B), abort flag (4 B), pad (8 B), unit ring (4 B each)
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 4 * NUNIT + 1024;  // + slack for 1024-byte alignment
  static_assert(SMEM <= 232448, "shared memory budget");
  static constexpr int TMEM_COLS = 512;
  static constexpr int TM_S = 0;                       // S_k at k * 128
  static constexpr int TM_O = 256;                     // O_k at 256 + k * D
};

constexpr float kRescaleThreshold = 8.0f;
// A quarter of the unmasked tiles' exponentials (2 of every 8 pairs) run on the
// FMA pipe instead of MUFU, which the softmax's exponentials otherwise keep busy
// about as long as the tensor cores run a tile's products.  2^x = 2^n 2^f with
// n = round(x), f = x - n in [-1/2, 1/2] (Cody-Waite reduction), 2^f by a cubic
// whose coefficients minimise the relative error on [-1/2, 1/2] with p(0) = 1
// (fit_exp2_poly.py, a linear programme; largest relative error 1.013e-4, far
// below the bf16 rounding of P).  x is first clamped to [-124, 132] through a
// saturated y = (x + 124) / 256, so that adding n to the exponent field of 2^f
// never leaves the normal range; clamping at -124 turns weights below 2^-124
// (invisible next to a row's largest, which is at least 2^-8) into 2^-124.
constexpr int kFmaPairsPer8 = 2;
constexpr float kExpC1 = 0.6932829022407532f, kExpC2 = 0.2422109693288803f, kExpC3 = 0.055009059607982635f;  // log2 units: weights stay below 256

enum : int {  // wait sites recorded in the device status word on a timeout
  kSiteFwdProducer = 0x101,
  kSiteFwdMmaQ = 0x102,
  kSiteFwdMmaK = 0x103,
  kSiteFwdMmaP = 0x105,
  kSiteFwdMmaV = 0x106,
  kSiteFwdSoftS = 0x107,
  kSiteFwdSoftO = 0x108,
  kSiteFwdMmaO = 0x109,
  kSiteFwdUnit = 0x10a,
};

template <int D, bool CAUSAL, bool DROPOUT>
__global__ void __launch_bounds__(384, 1)
    fattn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const FwdArgs args) {
  using C = FwdCfg<D>;
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);

  auto sQ = [&](int b) { return sbase + C::OFF_Q + b * C::TILE; };
  const uint32_t sSlot0 = sbase + C::OFF_SLOT;
  const uint32_t bar0 = sbase + C::OFF_BAR;
  auto bar = [&](int i) { return bar0 + 8u * i; };
  auto bar_q_full = [&](int b) { return bar(C::B_QF + b); };
  auto bar_q_empty = [&](int b) { return bar(C::B_QE + b); };
  auto bar_slot_full = [&](int s) { return bar(C::B_SF + s); };
  auto bar_slot_empty = [&](int s) { return bar(C::B_SE + s); };
  auto bar_s_full = [&](int k) { return bar(C::B_S + k); };
  auto bar_p_full = [&](int k) { return bar(C::B_P + k); };
  auto bar_pv_done = [&](int k) { return bar(C::B_PV + k); };
  auto bar_o_free = [&](int k) { return bar(C::B_OF + k); };
  const uint32_t bar_drain = bar(C::B_DRAIN);
  auto bar_unit_full = [&](int e) { return bar(C::B_UF + e); };
  auto bar_unit_empty = [&](int e) { return bar(C::B_UE + e); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  volatile int* unit_ring = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 16);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Work units.  Non-causal heads: batch*head slowest, then the pair of query
  // tiles; every unit costs the same.  Causal heads: the heads form groups of
  // group_big or group_big - 1; inside a group the longest pairs of all its heads
  // come first (longest-processing-time order), so the group's short units fill
  // in behind its long ones, while the group's keys and values stay in L2.
  const int NT = args.num_q_tiles;
  const int NKT = args.num_kv_tiles;
  const int NP = (NT + 1) >> 1;
  const bool dyn = CAUSAL && args.sched != nullptr;
  struct Unit {
    int bh, kv_bh, head_row0, tile0, n_kv0, n_kv1, n_kv;
  };
  auto unit_of = [&](int u) {
    Unit w;
    int bh, pair;
    if (CAUSAL) {
      const int big = args.group_big, ubig = NP * big, nbig_units = args.num_big_groups * ubig;
      int r, hg, h0;
      if (u < nbig_units) {
        const int g = u / ubig;
        r = u - g * ubig;
        hg = big;
        h0 = g * big;
      } else {
        const int gs = NP * (big - 1), u2 = u - nbig_units, g = u2 / gs;
        r = u2 - g * gs;
        hg = big - 1;
        h0 = args.num_big_groups * big + g * (big - 1);
      }
      bh = h0 + r % hg;
      pair = NP - 1 - r / hg;
    } else {
      bh = u / NP;
      pair = u % NP;
    }
    w.bh = bh;
    w.kv_bh = bh / args.G;  // b*H + h -> b*H_kv + h / G
    w.head_row0 = bh * args.N_q;
    w.tile0 = 2 * pair;
    const bool has_q1 = w.tile0 + 1 < NT;
    // key tiles each query tile needs (contiguous from 0); 0 = tile absent
    w.n_kv0 = fwd_kv_tiles(w.tile0, NKT, args.causal_off, CAUSAL);
    w.n_kv1 = has_q1 ? fwd_kv_tiles(w.tile0 + 1, NKT, args.causal_off, CAUSAL) : 0;
    w.n_kv = w.n_kv1 > w.n_kv0 ? w.n_kv1 : w.n_kv0;
    return w;
  };

  if (threadIdx.x == 0) {
    for (int b = 0; b < C::QBUF; ++b) {
      mbar_init(bar_q_full(b), 1);
      mbar_init(bar_q_empty(b), 1);
    }
    for (int s = 0; s < C::NSLOT; ++s) {
      mbar_init(bar_slot_full(s), 1);
      mbar_init(bar_slot_empty(s), 1);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(bar_s_full(k), 1);
      mbar_init(bar_p_full(k), 128);
      mbar_init(bar_pv_done(k), 1);
      mbar_init(bar_o_free(k), 128);
    }
    mbar_init(bar_drain, 1);
    for (int e = 0; e < C::NUNIT; ++e) {
      mbar_init(bar_unit_full(e), 1);
      mbar_init(bar_unit_empty(e), 1 + 8);  // the MMA thread and one lane of each softmax warp
    }
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
  // take 208, the producer/MMA group keeps 88: 2*128*208 + 128*88 = 64512.
  if (warp >= 8) {
    regs_decrease<88>();
    if (warp == 8) {
      // ------------------------------------------------------------ producer
      // The whole warp runs the loop and its waits; lane 0 alone issues the copies,
      // the barrier transactions and the unit claims (one()).  A lone lane running
      // the loop competes for issue slots with the softmax warps beside it.
      {
        auto one = [&](auto f) { if (lane == 0) f(); __syncwarp(); };
        one([&] {
          prefetch_tensormap(&tm_q);
          prefetch_tensormap(&tm_k);
          prefetch_tensormap(&tm_v);
        });
        int it = 0;  // K/V tiles loaded (ring position), continuous across units
        int qs = 0;  // Q tiles loaded (Q ring position)
        bool ok = true;
        int u = blockIdx.x;  // the first unit by block index
        for (int nu = 0; ok; ++nu) {
          const int e = nu % C::NUNIT;
          if (!(ok = mbar_wait(bar_unit_empty(e), ((nu / C::NUNIT) & 1) ^ 1, abort_flag, kSiteFwdUnit))) break;
          one([&] {
            unit_ring[e] = u < args.num_units ? u : -1;
            mbar_arrive(bar_unit_full(e));
          });
          if (u >= args.num_units) break;
          const Unit w = unit_of(u);
          const int nq = w.n_kv1 > 0 ? 2 : 1;
          unsigned int ticket = 0;
          for (int j = 0; j < w.n_kv && ok; ++j) {
            // A dynamic CTA claims its next unit as the loads of this unit's last
            // key/value tile go out: late enough that no CTA sits on a unit while
            // another has run out of work, early enough to hide the atomic.
            if (dyn && j == w.n_kv - 1) {
              unsigned int t = 0;
              if (lane == 0) t = atomicAdd(args.sched, 1u);
              ticket = __shfl_sync(0xffffffffu, t, 0);
            }
            for (int t = 0; t < 2 && ok; ++t) {
              const int s = it % C::NSLOT;
              if (!(ok = mbar_wait(bar_slot_empty(s), ((it / C::NSLOT) & 1) ^ 1, abort_flag, kSiteFwdProducer)))
                break;
              one([&] {
                mbar_arrive_expect_tx(bar_slot_full(s), C::TILE);
                const CUtensorMap* map = (t == 0) ? &tm_k : &tm_v;
                const uint32_t dst = sSlot0 + s * C::TILE;
#pragma unroll
                for (int kb = 0; kb < C::L::NB; ++kb)
                  tma_load_3d(dst + kb * C::L::BLKB, map, bar_slot_full(s), kb * C::L::CW, j * 128, w.kv_bh);
              });
              ++it;
              // Q0 after K_0, Q1 after V_0: each into the Q buffer freed longest ago
              if (j == 0 && t < nq) {
                const int b = qs % C::QBUF;
                if (!(ok = mbar_wait(bar_q_empty(b), ((qs / C::QBUF) & 1) ^ 1, abort_flag, kSiteFwdProducer)))
                  break;
                one([&] {
                  mbar_arrive_expect_tx(bar_q_full(b), C::TILE);
#pragma unroll
                  for (int kb = 0; kb < C::L::NB; ++kb)
                    tma_load_3d(sQ(b) + kb * C::L::BLKB, &tm_q, bar_q_full(b), kb * C::L::CW, (w.tile0 + t) * 128,
                                w.bh);
                });
                ++qs;
              }
            }
          }
          u = dyn ? (int)gridDim.x + (int)ticket : u + (int)gridDim.x;
        }
        if (!ok) {  // aborted: let the copies already issued land before the CTA exits
          for (int i = (qs > C::QBUF ? qs - C::QBUF : 0); i < qs; ++i)
            mbar_wait_ns(bar_q_full(i % C::QBUF), (i / C::QBUF) & 1, 100000000ull);
          for (int i = (it > C::NSLOT ? it - C::NSLOT : 0); i < it; ++i)
            mbar_wait_ns(bar_slot_full(i % C::NSLOT), (i / C::NSLOT) & 1, 100000000ull);
        }
      }
      __syncwarp();
    } else if (warp == 9) {
      // ----------------------------------------------------------- MMA issuer
      // The whole warp runs this loop; lane 0 issues each tcgen05 instruction
      // (mma_*_warp) and makes the plain arrivals.
      {
        constexpr uint32_t idS = idesc_bf16_f32(128, 128, false, false);  // Q (K-major) x K (K-major)
        constexpr uint32_t idPV = idesc_bf16_f32(128, D, false, true);    // P (TMEM) x V (MN-major)
        auto slot_of = [&](int i) { return i % C::NSLOT; };
        auto issue_s = [&](int k, int qbuf, int kslot) {  // S_k = Q K^T, Q from buffer qbuf, K from ring slot kslot
          // The start address is a descriptor's low 14 bits (address / 16, below
          // 2^14 for any shared-memory address), so each K step adds a constant to
          // one base descriptor per operand.  The bases pass through an opaque
          // move: hoisted out of the loops, the descriptors of every buffer and
          // step would not fit in this thread's registers.
          const uint64_t dq = C::L::desc_k(opaque_u32(sQ(qbuf)));
          const uint64_t dk = C::L::desc_k(opaque_u32(sSlot0 + kslot * C::TILE));
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off16 = C::L::kstep(kk) >> 4;
            mma_ss_warp(tmem + C::TM_S + k * 128, dq + off16, dk + off16, idS, kk > 0 ? 1u : 0u);
          }
          mma_commit_warp(bar_s_full(k));
        };
        int it = 0;          // ring position of the current unit's K_0
        int qs = 0;          // Q ring position of the current unit's Q0
        int tk[2] = {0, 0};  // tiles processed per query-tile slot (phases of s_full/p_full/pv_done)
        int uk[2] = {0, 0};  // units in which each query-tile slot was active (phases of o_free)
        bool ok = true;
        for (int nu = 0; ok; ++nu) {
          const int e = nu % C::NUNIT;
          if (!(ok = mbar_wait(bar_unit_full(e), (nu / C::NUNIT) & 1, abort_flag, kSiteFwdUnit))) break;
          const int u = unit_ring[e];
          if (lane == 0) mbar_arrive(bar_unit_empty(e));
          __syncwarp();
          if (u < 0) break;
          const Unit w = unit_of(u);
          const int nq = w.n_kv1 > 0 ? 2 : 1;
          const int it0 = it;
          auto n_kv_of = [&](int k) { return k == 0 ? w.n_kv0 : w.n_kv1; };
          auto qbuf = [&](int k) { return (qs + k) % C::QBUF; };
          // prologue: S_k(0).  S_k(0) of a unit overwrites the columns the previous
          // unit's last PV_k read P_k from; tcgen05.mma of one thread execute in
          // issue order.
          if (!(ok = mbar_wait(bar_slot_full(slot_of(it0)), (it0 / C::NSLOT) & 1, abort_flag, kSiteFwdMmaK))) break;
          for (int k = 0; k < nq && ok; ++k) {
            if (!(ok = mbar_wait(bar_q_full(qbuf(k)), ((qs + k) / C::QBUF) & 1, abort_flag, kSiteFwdMmaQ))) break;
            tc_fence_after();
            issue_s(k, qbuf(k), slot_of(it0));
            if (n_kv_of(k) == 1) mma_commit_warp(bar_q_empty(qbuf(k)));  // Q_k's only product
          }
          if (!ok) break;
          mma_commit_warp(bar_slot_empty(slot_of(it0)));
          // Issue order: S0_0 S1_0 | PV0_0 S0_1 | PV1_0 S1_1 | PV0_1 S0_2 | ...  While one
          // softmax group works on S_k, the tensor cores run the other group's P V and
          // its next S.  S_k(j+1) overwrites the columns PV_k(j) reads P_k(j) from.
          for (int j = 0; j < w.n_kv && ok; ++j) {
            const int itV = it0 + 2 * j + 1, itK1 = it0 + 2 * j + 2;
            if (!(ok = mbar_wait(bar_slot_full(slot_of(itV)), (itV / C::NSLOT) & 1, abort_flag, kSiteFwdMmaV)))
              break;
            const bool more = j + 1 < w.n_kv;
            if (more &&
                !(ok = mbar_wait(bar_slot_full(slot_of(itK1)), (itK1 / C::NSLOT) & 1, abort_flag, kSiteFwdMmaK)))
              break;
            const uint32_t vaddr = sSlot0 + slot_of(itV) * C::TILE;
            for (int k = 0; k < 2 && ok; ++k) {
              if (j >= n_kv_of(k)) continue;
              // the first P V of a unit overwrites O_k: the previous epilogue must have read it
              if (j == 0 && uk[k] > 0 &&
                  !(ok = mbar_wait(bar_o_free(k), (uk[k] - 1) & 1, abort_flag, kSiteFwdMmaO)))
                break;
              if (!(ok = mbar_wait(bar_p_full(k), tk[k] & 1, abort_flag, kSiteFwdMmaP))) break;
              tc_fence_after();
              const uint32_t tP = tmem + C::TM_S + k * 128;
              const uint64_t dv = C::L::desc_mn(opaque_u32(vaddr), C::L::BLKB);
#pragma unroll
              for (int kk = 0; kk < 8; ++kk)  // K = 128 keys, 16 per step = 8 TMEM columns of packed P
                mma_ts_warp(tmem + C::TM_O + k * D, tP + kk * 8, dv + kk * (C::L::ROWSTEP16 >> 4), idPV,
                       (j > 0 || kk > 0) ? 1u : 0u);
              mma_commit_warp(bar_pv_done(k));
              ++tk[k];
              if (j + 1 < n_kv_of(k)) {
                issue_s(k, qbuf(k), slot_of(itK1));
                if (j + 2 == n_kv_of(k)) mma_commit_warp(bar_q_empty(qbuf(k)));  // Q_k's last product
              }
            }
            if (!ok) break;
            mma_commit_warp(bar_slot_empty(slot_of(itV)));
            if (more) mma_commit_warp(bar_slot_empty(slot_of(itK1)));
          }
          it = it0 + 2 * w.n_kv;
          qs += nq;
          for (int k = 0; k < nq; ++k) ++uk[k];
        }
        // Make sure nothing this thread issued is still running before TMEM is freed.
        mma_commit_warp(bar_drain);
        mbar_wait_ns(bar_drain, 0, 100000000ull);
      }
      __syncwarp();
    }
  } else {
    regs_increase<208>();
    // ------------------------------------------------------ softmax groups
    const int k = warp >> 2;  // query-tile slot of this group
    const int wq = warp & 3;
    const int r = wq * 32 + lane;  // row inside the query tile
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tS = tmem + C::TM_S + k * 128 + lane_off;
    const uint32_t tO = tmem + C::TM_O + k * D + lane_off;
    const float sl2 = args.scale_log2;
    int tk = 0;  // tiles processed (phases of s_full/p_full/pv_done for this slot)
    bool ok = true;
    for (int nu = 0; ok; ++nu) {
      const int e = nu % C::NUNIT;
      ok = __all_sync(0xffffffffu, mbar_wait(bar_unit_full(e), (nu / C::NUNIT) & 1, abort_flag, kSiteFwdUnit));
      if (!ok) break;
      const int u = unit_ring[e];
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_unit_empty(e));
      if (u < 0) break;
      const Unit w = unit_of(u);
      const int n_kv_k = k == 0 ? w.n_kv0 : w.n_kv1;
      if (n_kv_k == 0) continue;  // no second query tile in this unit
      const int q_tile = w.tile0 + k;
      float m_ref = -INFINITY;  // reference max of the scaled scores, log2 units
      float l = 0.f;            // running sum of exp2(score - m_ref)
      for (int j = 0; j < n_kv_k; ++j, ++tk) {
        ok = mbar_wait(bar_s_full(k), tk & 1, abort_flag, kSiteFwdSoftS);
        if (!(ok = __all_sync(0xffffffffu, ok))) break;
        tc_fence_after();
        // S_k row r -> registers in two halves of 64 keys: the row max of the first
        // half runs while the second is still on its way from TMEM.  On the diagonal
        // tile the keys c > r become -inf (+inf for a negative scale) first.  Row max
        // of the raw scores, turned into the max of scale * score (log2 units); four
        // independent three-input chains keep the dependencies short.
        uint32_t v[4][32];
        // Keys c >= lim of this tile are masked.  Causal: key 128 j + c is visible to
        // query 128 q_tile + r iff 128 j + c <= 128 q_tile + r + off, so lim = base + r
        // with base = 128 (q_tile - j) + off + 1, and only tiles with base < 128
        // mask anything.  Non-causal: a ragged last key tile, whose keys c >= kv_tail
        // are past the sequence (their rows read as zero).  Causal rows never see
        // those: the mask hides every key past N_k from every query before N_q.
        const int base = 128 * (q_tile - j) + args.causal_off + 1;
        const bool clip = CAUSAL ? base < 128 : (j == NKT - 1 && args.kv_tail < 128);
        const int lim = CAUSAL ? base + r : args.kv_tail;
        // The mask is uniform over the tile, so the masked and the unmasked tiles
        // get their own copies of the unrolled loops, picked by one branch per
        // tile: a test inside the unrolled loops would be if-converted into compares
        // and selects that every tile pays for.
        const float masked = sl2 >= 0.f ? -INFINITY : INFINITY;
        float mx;
        tmem_ld32(tS, v[0]);
        tmem_ld32(tS + 32, v[1]);
        tmem_ld_wait(v[0]);
        tmem_ld_wait(v[1]);
        tmem_ld32(tS + 64, v[2]);
        tmem_ld32(tS + 96, v[3]);
        {
          float pm[4] = {masked, masked, masked, masked};
          auto half = [&](int h, auto clip_c) {
            if constexpr (decltype(clip_c)::value) {
  #pragma unroll
              for (int c = h * 64; c < h * 64 + 64; ++c)
                if (c >= lim) v[c >> 5][c & 31] = __float_as_uint(masked);
            }
            if (sl2 >= 0.f) {
  #pragma unroll
              for (int c = h * 64; c < h * 64 + 64; c += 8)
  #pragma unroll
                for (int u = 0; u < 4; ++u)
                  pm[u] = fmax3(pm[u], __uint_as_float(v[(c + 2 * u) >> 5][(c + 2 * u) & 31]),
                                __uint_as_float(v[(c + 2 * u + 1) >> 5][(c + 2 * u + 1) & 31]));
            } else {
  #pragma unroll
              for (int c = h * 64; c < h * 64 + 64; c += 8)
  #pragma unroll
                for (int u = 0; u < 4; ++u)
                  pm[u] = fmin3(pm[u], __uint_as_float(v[(c + 2 * u) >> 5][(c + 2 * u) & 31]),
                                __uint_as_float(v[(c + 2 * u + 1) >> 5][(c + 2 * u + 1) & 31]));
            }
          };
          if (clip) {
            half(0, std::true_type{});
            tmem_ld_wait(v[2]);
            tmem_ld_wait(v[3]);
            half(1, std::true_type{});
          } else {
            half(0, std::false_type{});
            tmem_ld_wait(v[2]);
            tmem_ld_wait(v[3]);
            half(1, std::false_type{});
          }
          mx = sl2 >= 0.f ? fmax3(pm[0], pm[1], fmaxf(pm[2], pm[3])) : fmin3(pm[0], pm[1], fminf(pm[2], pm[3]));
          mx *= sl2;
        }
        // lazily move the reference max; rescale O and l only when it moves
        const bool grow = mx > m_ref + kRescaleThreshold;
        if (__any_sync(0xffffffffu, grow)) {
          const float m_new = fmaxf(m_ref, mx);
          // 0 on a row's first visible keys (m_ref = -inf); 1 where the reference
          // stays, also while a row has seen no visible key (m_ref = m_new = -inf)
          const float alpha = m_new == m_ref ? 1.f : ex2(m_ref - m_new);
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
        // Keys c >= lim of this tile get weight 0, by a select after the exponential:
        // the masked raw scores were set to -inf (+inf for a negative scale), and
        // with scale 0 the product -inf * 0 is NaN, so the exponential alone cannot
        // be trusted to give 0.
        // Dropout (page 2's op chain: softmax, dropout, then V): the undropped
        // weights go into the row sum l, the dropped and rescaled ones into P V.
        // Without dropout the loop is instantiated with and without the mask, as
        // above; with dropout, whose keep bits already make it the longer loop, one
        // copy tests the mask per element (a second copy would spill).
        const uint32_t q_row = (uint32_t)(q_tile * 128 + r);
        const uint64_t sl2x2 = f2_pack(sl2, sl2), negm2 = f2_pack(-m_ref, -m_ref);
        const float pa = sl2 * (1.f / 256.f), pb = (124.f - m_ref) * (1.f / 256.f);  // y = s pa + pb
        uint32_t pk[2][32];  // P row as packed bf16 pairs
        auto exps = [&](auto mode_c) {
          constexpr int MODE = decltype(mode_c)::value;  // 0: no mask, 1: mask, 2: mask if clip
          uint32_t keep = 0xffffffffu;                    // keep bits of the current 32 keys
          uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};     // packed partial row sums
  #pragma unroll
          for (int c = 0; c < 128; c += 2) {
            const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(v[c >> 5][c & 31]),
                                               __uint_as_float(v[(c + 1) >> 5][(c + 1) & 31])),
                                       sl2x2, negm2);
            float p0, p1;
            if (MODE == 0 && ((c >> 1) & 7) < kFmaPairsPer8) {
              // y = sat((x + 124) / 256) stands for x; t = 1.5 * 2^23 + round(x) carries n
              // in its low bits; f = x - n; 2^f by the cubic; n added to the exponent
              const uint64_t y = f2_pack(fma_sat(__uint_as_float(v[c >> 5][c & 31]), pa, pb),
                                         fma_sat(__uint_as_float(v[(c + 1) >> 5][(c + 1) & 31]), pa, pb));
              const uint64_t t = f2_fma(y, f2_pack(256.f, 256.f), f2_pack(12582912.f - 124.f, 12582912.f - 124.f));
              const uint64_t w2 = f2_fma(t, f2_pack(-1.f, -1.f), f2_pack(12582912.f - 124.f, 12582912.f - 124.f));
              const uint64_t f = f2_fma(y, f2_pack(256.f, 256.f), w2);
              uint64_t q = f2_fma(f, f2_pack(kExpC3, kExpC3), f2_pack(kExpC2, kExpC2));
              q = f2_fma(q, f, f2_pack(kExpC1, kExpC1));
              q = f2_fma(q, f, f2_pack(1.f, 1.f));
              float q0, q1, t0, t1;
              f2_unpack(q, q0, q1);
              f2_unpack(t, t0, t1);
              p0 = __uint_as_float(imad_u32(__float_as_uint(t0), 1u << 23, __float_as_uint(q0)));
              p1 = __uint_as_float(imad_u32(__float_as_uint(t1), 1u << 23, __float_as_uint(q1)));
            } else {
              float x0, x1;
              f2_unpack(x2, x0, x1);
              p0 = ex2(x0);
              p1 = ex2(x1);
            }
            if (MODE == 1 || (MODE == 2 && clip)) {
              p0 = (c < lim) ? p0 : 0.f;
              p1 = (c + 1 < lim) ? p1 : 0.f;
            }
            acc[(c >> 1) & 3] = f2_add(acc[(c >> 1) & 3], f2_pack(p0, p1));
            if constexpr (DROPOUT) {
              if ((c & 31) == 0) {
                keep = 0;
  #pragma unroll
                for (int u = 0; u < 8; ++u)  // keys c .. c + 31, four per generator call
                  keep |= dropout_keep4(args.drop, (uint32_t)w.bh, q_row, (uint32_t)((j * 128 + c) / 4 + u))
                          << (4 * u);
              }
              const float ks = args.drop.scale_keep;
              p0 = ((keep >> (c & 31)) & 1u) ? p0 * ks : 0.f;
              p1 = ((keep >> ((c + 1) & 31)) & 1u) ? p1 * ks : 0.f;
            }
            pk[c >> 6][(c >> 1) & 31] = pack_bf16x2(p0, p1);
          }
          const uint64_t a2 = f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3]));
          float s0, s1;
          f2_unpack(a2, s0, s1);
          l += s0 + s1;
        };
        if constexpr (DROPOUT) {
          exps(std::integral_constant<int, 2>{});
        } else {
          if (clip)
            exps(std::integral_constant<int, 1>{});
          else
            exps(std::integral_constant<int, 0>{});
        }
        // P (bf16 pairs) over the first 64 columns of S_k
        tmem_st32(tS, pk[0]);
        tmem_st32(tS + 32, pk[1]);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar_p_full(k));
      }
      if (!ok) break;
      ok = __all_sync(0xffffffffu, mbar_wait(bar_pv_done(k), (tk - 1) & 1, abort_flag, kSiteFwdSoftO));
      if (!ok) break;
      tc_fence_after();
      uint32_t o[D / 32][32];
#pragma unroll
      for (int c = 0; c < D / 32; ++c) tmem_ld32(tO + c * 32, o[c]);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) tmem_ld_wait(o[c]);
      tc_fence_before();
      mbar_arrive(bar_o_free(k));  // O_k may now be overwritten by the next unit
      // O row (bf16) straight to global memory, LSE (natural log) beside it; rows
      // of a ragged last tile past the sequence are not written
      if (q_tile * 128 + r < args.N_q) {
        const float inv_l = l > 0.f ? 1.f / l : 0.f;  // a row with no visible key: O = 0
        const size_t row = (size_t)(w.head_row0 + q_tile * 128 + r);
        uint4* dst = reinterpret_cast<uint4*>(args.o + row * D);
#pragma unroll
        for (int c = 0; c < D / 32; ++c)
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const uint32_t* x = &o[c][q4 * 8];
            dst[c * 4 + q4] = make_uint4(pack_bf16x2(__uint_as_float(x[0]) * inv_l, __uint_as_float(x[1]) * inv_l),
                                         pack_bf16x2(__uint_as_float(x[2]) * inv_l, __uint_as_float(x[3]) * inv_l),
                                         pack_bf16x2(__uint_as_float(x[4]) * inv_l, __uint_as_float(x[5]) * inv_l),
                                         pack_bf16x2(__uint_as_float(x[6]) * inv_l, __uint_as_float(x[7]) * inv_l));
          }
        args.lse[row] = (m_ref + __log2f(l)) * 0.69314718055994530942f;
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
  if (dyn && threadIdx.x == 0) {
    // the last CTA to finish returns both counters to 0 for the next launch
    __threadfence();
    if (atomicAdd(args.sched + 1, 1u) == gridDim.x - 1) {
      atomicExch(args.sched, 0u);
      atomicExch(args.sched + 1, 0u);
      __threadfence();
    }
  }
}

}  // namespace fattn
