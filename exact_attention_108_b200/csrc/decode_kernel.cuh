// decode_kernel.cuh -- split-KV attention for incremental decoding (sm_100a).
//
// Inference appends a few query rows at a time to a long sequence whose keys and
// values sit in a cache; its cost is reading that cache (page 2 "落地使用时应关注
// 什么": training and incremental inference are bound by different things; page 1
// "五、行业应用与演进方向": long-sequence inference).  The work per query row is
// too small to fill the GPU with one CTA per query tile, so
//   * the G = H / H_kv query heads that share a key/value head are packed into one
//     tile: their G * N_q rows are contiguous in memory ([B, H, N_q, d] with the
//     heads of a group adjacent), so a 3-D tensor map views q as
//     [B*H_kv][G*N_q][d] and one 128-row tile holds up to 128 of them;
//   * each (key/value head, row tile) is split into key ranges, one CTA each, so
//     that B * H_kv * splits CTAs stream the cache at full HBM bandwidth.
// Every CTA runs the same online softmax as the forward over its key range
// (page 3 "4.2 在线softmax技巧") and writes its rows' partial result: O divided by
// its own row sum and its log-sum-exp (log2 units).  fattn_decode_merge_kernel
// then combines the splits of a row with weights 2^(lse_s - max_s lse_s).  With
// one split the CTA writes the final bf16 O and natural-log LSE itself.
//
// Roles (192 threads): warps 0..3 softmax (thread = packed row), warp 4 TMA
// producer (Q once, K_j, V_j through an NSLOT-deep ring), warp 5 tcgen05 issuer (the
// whole warp; lane 0 issues each instruction).
// S goes to two TMEM buffers (columns 0 and 128), so S_{j+1} runs while the
// softmax works on S_j; O accumulates at column 256.  Warps whose 32 rows are all
// padding skip the exponentials: their P rows only feed output rows that are
// never stored.
#pragma once

#include <type_traits>

#include "sm100.cuh"

namespace fattn {

struct DecodeArgs {
  float* o_part;        // [splits][B*H_kv][rows][D] fp32, normalised (splits > 1)
  float* lse_part;      // [splits][B*H_kv][rows] fp32, log2 units (splits > 1)
  __nv_bfloat16* o;     // [B*H*N_q, D] bf16 (splits == 1)
  float* lse;           // [B*H*N_q] fp32, natural log (splits == 1)
  int rows;             // G * N_q: packed rows per key/value head
  int row_tiles;        // RT = ceil(rows / 128)
  int N_q, N_k;
  int num_kv_tiles;     // ceil(N_k / 128)
  int tiles_per_split;
  int splits;
  int kv_heads;         // B * H_kv
  int causal_off;       // N_k - N_q
  float scale_log2;
};

template <int D>
struct DecodeCfg {
  using L = sm100::Cols<D>;
  static constexpr int TILE = 128 * D * 2;
  static constexpr int NSLOT = D == 256 ? 2 : D == 128 ? 6 : D == 96 ? 8 : D == 64 ? 12 : 16;
  static constexpr int OFF_Q = 0, OFF_SLOT = TILE;
  static constexpr int OFF_BAR = OFF_SLOT + NSLOT * TILE;
  // q_full, slot_full[NSLOT], slot_empty[NSLOT], s_full[2], p_full[2], pv_done, o_done, drain
  static constexpr int B_Q = 0, B_SF = 1, B_SE = 1 + NSLOT, B_S = 1 + 2 * NSLOT, B_P = B_S + 2;
  static constexpr int B_PV = B_P + 2, B_OD = B_PV + 1, B_DRAIN = B_PV + 2, NBAR = B_DRAIN + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = OFF_MISC + 16;
  static_assert(SMEM <= 232448, "shared memory budget");
  static constexpr int TMEM_COLS = 512;
  static constexpr int TM_S = 0, TM_O = 256;
};

enum : int {
  kSiteDecProducer = 0x401,
  kSiteDecMmaQ = 0x402,
  kSiteDecMmaK = 0x403,
  kSiteDecMmaV = 0x404,
  kSiteDecMmaP = 0x405,
  kSiteDecSoftS = 0x406,
  kSiteDecSoftO = 0x407,
  kSiteDecAlign = 0x408,
};

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(192, 1)
    fattn_decode_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const DecodeArgs args) {
  using C = DecodeCfg<D>;
  using namespace sm100;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_addr(smem);
  const uint32_t sQ = sbase + C::OFF_Q, sSlot0 = sbase + C::OFF_SLOT;
  const uint32_t bar0 = sbase + C::OFF_BAR;
  auto bar = [&](int i) { return bar0 + 8u * i; };
  const uint32_t bar_q_full = bar(C::B_Q);
  auto bar_slot_full = [&](int s) { return bar(C::B_SF + s); };
  auto bar_slot_empty = [&](int s) { return bar(C::B_SE + s); };
  auto bar_s_full = [&](int b) { return bar(C::B_S + b); };
  // p_full has one barrier per S buffer: warps whose rows are all padding pass a tile
  // at once, and with a single barrier their arrivals for tile j + 1 could complete
  // tile j's phase before the warp with real rows had written P_j
  auto bar_p_full = [&](int b) { return bar(C::B_P + b); };
  const uint32_t bar_pv_done = bar(C::B_PV), bar_o_done = bar(C::B_OD), bar_drain = bar(C::B_DRAIN);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (sbase & 1023u) {  // the swizzled layouts need 1024-byte alignment; never expected
    if (threadIdx.x == 0) atomicCAS(&g_fattn_status, 0, kSiteDecAlign);
    return;
  }
  // blockIdx.x = (split * kv_heads + kv head) * row_tiles + row tile
  const int rt = (int)(blockIdx.x % (unsigned)args.row_tiles);
  const int hb = (int)((blockIdx.x / (unsigned)args.row_tiles) % (unsigned)args.kv_heads);
  const int split = (int)(blockIdx.x / ((unsigned)args.row_tiles * (unsigned)args.kv_heads));
  const int j0 = split * args.tiles_per_split;
  int j1 = min(args.num_kv_tiles, j0 + args.tiles_per_split);
  if (CAUSAL) {
    // only the key tiles some row of this tile sees: up to key max_i + off, max_i the
    // largest query index among the tile's packed rows (g * N_q + i)
    const int p_first = rt * 128, p_last = min(args.rows, p_first + 128) - 1;
    const int max_i = p_first / args.N_q != p_last / args.N_q ? args.N_q - 1 : p_last % args.N_q;
    const int key_end = min(args.N_k, max_i + args.causal_off + 1);
    j1 = min(j1, key_end <= 0 ? 0 : (key_end + 127) / 128);
  }
  // >= 1: a range whose rows see no key still runs one fully masked tile, so that its
  // O = 0 and LSE = -inf are written
  const int n_kv = max(1, j1 - j0);

  if (threadIdx.x == 0) {
    mbar_init(bar_q_full, 1);
    for (int s = 0; s < C::NSLOT; ++s) {
      mbar_init(bar_slot_full(s), 1);
      mbar_init(bar_slot_empty(s), 1);
    }
    mbar_init(bar_s_full(0), 1);
    mbar_init(bar_s_full(1), 1);
    mbar_init(bar_p_full(0), 128);
    mbar_init(bar_p_full(1), 128);
    mbar_init(bar_pv_done, 1);
    mbar_init(bar_o_done, 1);
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_addr(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    // The whole warp runs the loop and its waits; lane 0 alone issues the copies
    // and the barrier transactions (one()).
    {
      auto one = [&](auto f) { if (lane == 0) f(); __syncwarp(); };
      one([&] {
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
        mbar_arrive_expect_tx(bar_q_full, C::TILE);
#pragma unroll
        for (int kb = 0; kb < C::L::NB; ++kb)
          tma_load_3d(sQ + kb * C::L::BLKB, &tm_q, bar_q_full, kb * C::L::CW, rt * 128, hb);
      });
      int it = 0;  // K_j at 2j, V_j at 2j + 1 (j counted from the split's first tile)
      bool ok = true;
      for (int j = 0; j < n_kv && ok; ++j) {
        for (int t = 0; t < 2 && ok; ++t, ++it) {
          const int s = it % C::NSLOT;
          if (!(ok = mbar_wait(bar_slot_empty(s), ((it / C::NSLOT) & 1) ^ 1, abort_flag, kSiteDecProducer))) break;
          one([&] {
            mbar_arrive_expect_tx(bar_slot_full(s), C::TILE);
            const CUtensorMap* map = t == 0 ? &tm_k : &tm_v;
#pragma unroll
            for (int kb = 0; kb < C::L::NB; ++kb)
              tma_load_3d(sSlot0 + s * C::TILE + kb * C::L::BLKB, map, bar_slot_full(s), kb * C::L::CW,
                          (j0 + j) * 128, hb);
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
  } else if (warp == 5) {
    // ---------------------------------------------------------- MMA issuer
    // The whole warp runs this loop; lane 0 issues each tcgen05 instruction
    // (mma_*_warp).
    {
      constexpr uint32_t idS = idesc_bf16_f32(128, 128, false, false);  // Q (K-major) x K (K-major)
      constexpr uint32_t idPV = idesc_bf16_f32(128, D, false, true);    // P (TMEM) x V (MN-major)
      auto slot_addr = [&](int i) { return sSlot0 + (i % C::NSLOT) * C::TILE; };
      auto wait_slot = [&](int i, int site) {
        return mbar_wait(bar_slot_full(i % C::NSLOT), (i / C::NSLOT) & 1, abort_flag, site);
      };
      auto issue_s = [&](int j) {  // S_j = Q K_j^T into buffer j & 1
        const uint64_t dq = C::L::desc_k(opaque_u32(sQ)), dk = C::L::desc_k(opaque_u32(slot_addr(2 * j)));
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off16 = C::L::kstep(kk) >> 4;
          mma_ss_warp(tmem + C::TM_S + (j & 1) * 128, dq + off16, dk + off16, idS, kk > 0 ? 1u : 0u);
        }
        mma_commit_warp(bar_s_full(j & 1));
        mma_commit_warp(bar_slot_empty((2 * j) % C::NSLOT));  // K_j has been read
      };
      bool ok = mbar_wait(bar_q_full, 0, abort_flag, kSiteDecMmaQ);
      for (int j = 0; j < 2 && j < n_kv && ok; ++j) {
        if (!(ok = wait_slot(2 * j, kSiteDecMmaK))) break;
        tc_fence_after();
        issue_s(j);
      }
      for (int j = 0; j < n_kv && ok; ++j) {
        // O += P_j V_j (P_j, bf16, over the first 64 columns of S buffer j & 1)
        if (!(ok = mbar_wait(bar_p_full(j & 1), (j >> 1) & 1, abort_flag, kSiteDecMmaP))) break;
        if (!(ok = wait_slot(2 * j + 1, kSiteDecMmaV))) break;
        tc_fence_after();
        const uint32_t tP = tmem + C::TM_S + (j & 1) * 128;
        const uint64_t dv = C::L::desc_mn(opaque_u32(slot_addr(2 * j + 1)), C::L::BLKB);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts_warp(tmem + C::TM_O, tP + kk * 8, dv + kk * (C::L::ROWSTEP16 >> 4), idPV, (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit_warp(bar_pv_done);
        mma_commit_warp(bar_slot_empty((2 * j + 1) % C::NSLOT));
        // S_{j+2} over buffer j & 1: P_j V_j, issued just before, reads it first
        if (j + 2 < n_kv) {
          if (!(ok = wait_slot(2 * j + 4, kSiteDecMmaK))) break;
          tc_fence_after();
          issue_s(j + 2);
        }
      }
      if (ok) mma_commit_warp(bar_o_done);  // every P_j V_j is in O
      mma_commit_warp(bar_drain);
      mbar_wait_ns(bar_drain, 0, 100000000ull);
    }
    __syncwarp();
  } else if (warp < 4) {
    // ------------------------------------------------------------- softmax
    const int r = warp * 32 + lane;  // packed row of the tile
    const int prow = rt * 128 + r;   // packed row of the key/value head: query head g, query i
    const bool warp_live = warp * 32 + rt * 128 < args.rows;  // some row of this warp is real
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const uint32_t tO = tmem + C::TM_O + lane_off;
    const float sl2 = args.scale_log2;
    // keys visible to this row: all N_k, or (causal) those up to i + N_k - N_q
    const int i_q = prow % args.N_q;
    const int key_end = CAUSAL ? min(args.N_k, i_q + args.causal_off + 1) : args.N_k;
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const uint32_t tS = tmem + C::TM_S + (j & 1) * 128 + lane_off;
      ok = mbar_wait(bar_s_full(j & 1), (j >> 1) & 1, abort_flag, kSiteDecSoftS);
      if (!(ok = __all_sync(0xffffffffu, ok))) break;
      tc_fence_after();
      if (warp_live) {
        const int lim = key_end - (j0 + j) * 128;  // keys c >= lim of this tile are masked
        const bool clip = __any_sync(0xffffffffu, lim < 128);
        const float masked = sl2 >= 0.f ? -INFINITY : INFINITY;
        uint32_t v[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32 * c, v[c]);
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld_wait(v[c]);
        float pm[4] = {masked, masked, masked, masked};
        auto mask_max = [&](auto clip_c) {
          if constexpr (decltype(clip_c)::value) {
#pragma unroll
            for (int c = 0; c < 128; ++c)
              if (c >= lim) v[c >> 5][c & 31] = __float_as_uint(masked);
          }
          if (sl2 >= 0.f) {
#pragma unroll
            for (int c = 0; c < 128; c += 8)
#pragma unroll
              for (int u = 0; u < 4; ++u)
                pm[u] = fmax3(pm[u], __uint_as_float(v[(c + 2 * u) >> 5][(c + 2 * u) & 31]),
                              __uint_as_float(v[(c + 2 * u + 1) >> 5][(c + 2 * u + 1) & 31]));
          } else {
#pragma unroll
            for (int c = 0; c < 128; c += 8)
#pragma unroll
              for (int u = 0; u < 4; ++u)
                pm[u] = fmin3(pm[u], __uint_as_float(v[(c + 2 * u) >> 5][(c + 2 * u) & 31]),
                              __uint_as_float(v[(c + 2 * u + 1) >> 5][(c + 2 * u + 1) & 31]));
          }
        };
        if (clip)
          mask_max(std::true_type{});
        else
          mask_max(std::false_type{});
        float mx = sl2 >= 0.f ? fmax3(pm[0], pm[1], fmaxf(pm[2], pm[3])) : fmin3(pm[0], pm[1], fminf(pm[2], pm[3]));
        mx *= sl2;
        // the reference max moves only when a row max exceeds it by more than 2^8
        const bool grow = mx > m_ref + 8.0f;
        if (__any_sync(0xffffffffu, grow)) {
          const float m_new = fmaxf(m_ref, mx);
          const float alpha = m_new == m_ref ? 1.f : ex2(m_ref - m_new);
          l *= alpha;
          m_ref = m_new;
          if (j > 0) {
            // O holds P_{j-1} V_{j-1} once that product is done.  The parity wait is
            // unambiguous: S_j was issued after P_{j-2} V_{j-2}, so that product is done
            // and pv_done has completed j - 1 or j phases.
            ok = __all_sync(0xffffffffu, mbar_wait(bar_pv_done, (j - 1) & 1, abort_flag, kSiteDecSoftO));
            if (!ok) break;
            tc_fence_after();
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
        const uint64_t sl2x2 = f2_pack(sl2, sl2), negm2 = f2_pack(-m_ref, -m_ref);
        uint32_t pk[2][32];
        // two copies of the unrolled loop, with and without the mask, picked once per
        // tile (a test inside the loop would be paid for as selects on every tile)
        auto exps = [&](auto clip_c) {
          uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
          for (int c = 0; c < 128; c += 2) {
            const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(v[c >> 5][c & 31]),
                                               __uint_as_float(v[(c + 1) >> 5][(c + 1) & 31])),
                                       sl2x2, negm2);
            float x0, x1;
            f2_unpack(x2, x0, x1);
            float p0 = ex2(x0), p1 = ex2(x1);
            if constexpr (decltype(clip_c)::value) {  // a select, not the exponential, zeroes
              p0 = c < lim ? p0 : 0.f;                // masked keys (-inf * 0 at scale 0)
              p1 = c + 1 < lim ? p1 : 0.f;
            }
            acc[(c >> 1) & 3] = f2_add(acc[(c >> 1) & 3], f2_pack(p0, p1));
            pk[c >> 6][(c >> 1) & 31] = pack_bf16x2(p0, p1);
          }
          const uint64_t a2 = f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3]));
          float s0, s1;
          f2_unpack(a2, s0, s1);
          l += s0 + s1;
        };
        if (clip)
          exps(std::true_type{});
        else
          exps(std::false_type{});
        tmem_st32(tS, pk[0]);
        tmem_st32(tS + 32, pk[1]);
        tmem_st_wait();
      }
      tc_fence_before();
      mbar_arrive(bar_p_full(j & 1));
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_o_done, 0, abort_flag, kSiteDecSoftO));
    if (ok && warp_live) {
      tc_fence_after();
      const bool row_ok = prow < args.rows;
      const float inv_l = l > 0.f ? 1.f / l : 0.f;  // a row with no visible key in this range: 0
      const float lse2 = m_ref + __log2f(l);         // -inf for such a row
      // O row, 32 columns at a time (a d = 256 row would not fit in registers at once):
      // bf16 to O with one split, else fp32 to this split's partial
      const size_t row = (size_t)hb * args.rows + prow;  // packed row (g, i) of key/value head hb
      const size_t prow_all = ((size_t)split * args.kv_heads + hb) * args.rows + prow;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + c * 32, o);
        tmem_ld_wait(o);
        if (!row_ok) continue;
        if (args.splits == 1) {
          uint4* dst = reinterpret_cast<uint4*>(args.o + row * D + c * 32);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const uint32_t* x = &o[q4 * 8];
            dst[q4] = make_uint4(pack_bf16x2(__uint_as_float(x[0]) * inv_l, __uint_as_float(x[1]) * inv_l),
                                 pack_bf16x2(__uint_as_float(x[2]) * inv_l, __uint_as_float(x[3]) * inv_l),
                                 pack_bf16x2(__uint_as_float(x[4]) * inv_l, __uint_as_float(x[5]) * inv_l),
                                 pack_bf16x2(__uint_as_float(x[6]) * inv_l, __uint_as_float(x[7]) * inv_l));
          }
        } else {
          float4* dst = reinterpret_cast<float4*>(args.o_part + prow_all * D + c * 32);
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) {
            const uint32_t* x = &o[q4 * 4];
            dst[q4] = make_float4(__uint_as_float(x[0]) * inv_l, __uint_as_float(x[1]) * inv_l,
                                  __uint_as_float(x[2]) * inv_l, __uint_as_float(x[3]) * inv_l);
          }
        }
      }
      if (row_ok) {
        if (args.splits == 1)
          args.lse[row] = lse2 * 0.69314718055994530942f;
        else
          args.lse_part[prow_all] = lse2;
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// Combines the splits of every packed row: with L_s the split's log2-sum-exp and
// O_s its normalised output, O = sum_s 2^(L_s - M) O_s / sum_s 2^(L_s - M) and
// LSE = (M + log2 sum_s 2^(L_s - M)) ln 2, M = max_s L_s.  A row that sees no key
// in any split (every L_s = -inf) gets O = 0 and LSE = -inf.  One warp per row,
// lane = D / 32 consecutive columns.
template <int D>
__global__ void __launch_bounds__(256) fattn_decode_merge_kernel(const DecodeArgs args) {
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);  // (kv head, packed row)
  const int lane = threadIdx.x & 31;
  if (row >= (long long)args.kv_heads * args.rows) return;
  const int hb = (int)(row / args.rows), prow = (int)(row % args.rows);
  const size_t stride = (size_t)args.kv_heads * args.rows;  // rows between splits
  const size_t base = (size_t)hb * args.rows + prow;
  float m = -INFINITY;
  for (int s = 0; s < args.splits; ++s) m = fmaxf(m, args.lse_part[base + s * stride]);
  constexpr int PER = D / 32;  // columns per lane: 1 to 8
  float acc[PER] = {};
  float wsum = 0.f;
  if (m != -INFINITY) {
    for (int s = 0; s < args.splits; ++s) {
      const float L = args.lse_part[base + s * stride];
      const float w = sm100::ex2(L - m);  // 0 for a split where the row sees no key
      wsum += w;
      const float* src = args.o_part + (base + s * stride) * D + lane * PER;
#pragma unroll
      for (int c = 0; c < PER; ++c) acc[c] = fmaf(w, src[c], acc[c]);
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  __nv_bfloat16* dst = args.o + ((size_t)hb * args.rows + prow) * D + lane * PER;
#pragma unroll
  for (int c = 0; c < PER; ++c) dst[c] = __float2bfloat16_rn(acc[c] * inv);
  if (lane == 0) args.lse[(size_t)hb * args.rows + prow] = (m + __log2f(wsum)) * 0.69314718055994530942f;
}

}  // namespace fattn
