// mla_pair_kernel.cuh -- absorbed-MLA decode on pairs of SMs.
//
// In MLA decode after absorption ("Full 路线" sections 4.2-4.3) every query
// head reads the same cached rows [c_kv (512) | k_pe (64)]; V is the first
// 512 columns of those rows.  With 128 heads the work is a dense contraction
// per key (2 * 128 * (576 + 512) flops per 1152 cached bytes), so one SM
// cannot keep up with HBM unless each cached byte crosses into shared memory
// about once: a single SM has room neither for Q^T of all 128 heads next to
// a K tile, nor for a 512 x 128 fp32 O^T in its 512 TMEM columns.
//
// A cluster of two CTAs on two SMs therefore works as one unit (tcgen05
// cta_group::2), on pair tiles of 256 keys of one sequence:
//
//   S^T[256 keys x 128 heads] = K[256 x 576] * Q^T       M = 256 keys: CTA r
//       holds keys 128r..128r+127 (its own K rows, loaded once); B = Q^T
//       split by heads: CTA r holds heads 64r..64r+63.  Each CTA's TMEM gets
//       S^T of its own 128 keys for all 128 heads.
//   softmax over keys per head: each CTA reduces its 128 keys, the two CTAs
//       exchange per-head tile maxima (st.async into the other CTA's shared
//       memory) so that both use the same running maximum.
//   O^T[512 x 128] += V^T[512 x 256 keys] * P^T[256 keys x 128 heads]
//       two pair MMAs (d rows 0..255 and 256..511, M = 256): CTA r provides
//       d rows 256m + 128r .. +127 of block m (two 64-column chunks of V for
//       all 256 keys) and P^T for its 64 heads; each CTA writes the P^T rows
//       of its own keys for the other CTA's heads into that CTA's buffer.
//       Each CTA's TMEM holds its 2 x 128 rows of O^T for all heads.
//
// Per pair tile each CTA copies 147 KB of K and 128 KB of V (the other CTA's
// V half comes from L2) in 32 KB boxes, a quarter of the copies per unit of
// work of one SM handling 64 heads.  Scheduling (persistent key ranges,
// pieces, workspace slots) is the split-KV decode's with 256-key tiles; the
// combine kernel merges the pieces.
//
// Roles (320 threads per CTA): warp 0 lane 0 streams K/V groups, lane 1
// loads this CTA's Q^T half per piece; warp 1 allocates the pair's TMEM and,
// in CTA 0, issues the pair UMMAs, in CTA 1 tells CTA 0 when its P^T buffer
// is complete; warps 2-9 run the softmax (two threads per key row, 64 heads
// each) and the epilogue.  All waits are bounded; the CTAs meet in a
// hardware cluster barrier only after both have left every loop.
//
// Gather mode (top-k decode, 384 threads): the keys of a sequence are the
// cache rows at caller-selected positions.  Warp 0 lane 0 is idle; warps
// 10-11 fill the same ring groups in the same order with 16-byte cp.async
// copies of the selected rows (so each selected byte crosses HBM once),
// and in CTA 1 warp 10 forwards each group's arrival to CTA 0.
//
// Cross-CTA traffic avoids cluster-scope release arrivals, which stall the
// arriving thread for about a microsecond while the SM streams copies: data
// (tile maxima, row sums, P^T rows) goes by st.async, whose bytes complete
// an mbarrier of the receiving CTA; signals without data (S^T read) are
// relaxed arrivals; MMA completions are tcgen05.commit multicasts.
#pragma once

#include "decode_kernel.cuh"

namespace attn {

struct MlaPairTraits {
  static constexpr int DK = 576, DV = 512;
  static constexpr int NH = 128;                  // heads per pair
  static constexpr int NHC = 64;                  // heads per CTA (Q^T rows, P^T columns)
  static constexpr int TILE = 128;                // keys per CTA per pair tile
  static constexpr int TILE_SHIFT = 8;            // 256 keys per pair tile
  static constexpr int KCH = DK / 64;             // 9 K chunks per row
  static constexpr int SLOT = 16384;              // [128 x 64] chunk
  static constexpr int GBYTES = 2 * SLOT;         // one copy: two chunks
  static constexpr int RING_G = 3;
  static constexpr int QT_CHUNK = NHC * 128;      // [64 heads x 64 columns]
  static constexpr int QT_BYTES = KCH * QT_CHUNK;
  static constexpr int PT_BYTES = 2 * TILE * NHC * 2;  // [256 keys x 64 heads] bf16
  static constexpr int OFF_RING = 0;
  static constexpr int OFF_QT = OFF_RING + RING_G * GBYTES;
  static constexpr int OFF_PT = OFF_QT + QT_BYTES;
  static constexpr int OFF_RED = OFF_PT + PT_BYTES;        // float [2][4][NH]
  static constexpr int OFF_PMAX = OFF_RED + 2 * 4 * NH * 4; // float [2][NH] peer tile maxima
  static constexpr int OFF_M = OFF_PMAX + 2 * NH * 4;       // float [NH] running max
  static constexpr int OFF_ALPHA = OFF_M + NH * 4;          // float [NH]
  static constexpr int OFF_L = OFF_ALPHA + NH * 4;          // float [NH] final sums
  static constexpr int OFF_LPEER = OFF_L + NH * 4;          // float [NH] peer sums
  static constexpr int OFF_SCAN = OFF_LPEER + NH * 4;       // int64 [8]
  static constexpr int OFF_SCHED = OFF_SCAN + 64;           // int [4]
  static constexpr int OFF_POS = OFF_SCHED + 16;            // int64 [4] range position
  static constexpr int OFF_FLAGS = OFF_POS + 32;            // int [4]: any[2], abort, tmem
  static constexpr int OFF_MERGE = OFF_FLAGS + 16;          // int: this CTA merges a unit half
  static constexpr int OFF_BAR = (OFF_MERGE + 16 + 7) & ~7;
  // full[3] empty[3] q_full q_free s_full[2] s_free[2] p_local p_recv p_peer o_done
  // red_full[2] stat_ready[2] xmax_full[2] lsum_full drain mg_done mg_flag
  static constexpr int NBAR = 2 * RING_G + 2 + 2 + 2 + 3 + 1 + 2 + 2 + 2 + 1 + 1 + 2;
  static constexpr int PT_PEER_BYTES = TILE * NHC * 2;     // P^T rows one CTA sends the other
  static constexpr int SMEM_BYTES = OFF_BAR + NBAR * 8 + 1024;
  static constexpr int SOFTMAX_THREADS = 256;
  static constexpr int THREADS = 64 + SOFTMAX_THREADS;
  // Top-k mode (rows gathered in the kernel): warps 10-11 copy the selected
  // rows; in CTA 1 warp 10 also forwards their arrival to CTA 0 (12 warps
  // keep the softmax warps' register budget of the dense kernel).
  static constexpr int GATHER_WARP0 = THREADS / 32;   // 10
  static constexpr int GATHER_THREADS = 64;
  static constexpr int THREADS_GATHER = THREADS + GATHER_THREADS;
  static constexpr int TMEM_S = 0;    // S^T double buffer: 2 x 128 columns
  static constexpr int TMEM_O = 256;  // O^T blocks m = 0, 1: 128 columns each
  static_assert(OFF_QT % 1024 == 0 && OFF_PT % 1024 == 0, "operand alignment");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

// Sum over the 32 lanes for each of N values per lane, transposed like
// transposed_warp_max: afterwards lane l holds in v[0 .. N/32 - 1] the sums
// of heads transposed_head<N>(l, i).
template <int NV, int N, int OFF>
__device__ __forceinline__ void transposed_warp_sum(float (&v)[NV], int lane) {
  if constexpr (OFF > 0) {
    constexpr int H = N / 2;
    const bool upper = (lane & OFF) != 0;
#pragma unroll
    for (int i = 0; i < H; ++i) {
      const float keep = upper ? v[i + H] : v[i];
      const float send = upper ? v[i] : v[i + H];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, OFF);
    }
    transposed_warp_sum<NV, H, OFF / 2>(v, lane);
  }
}

template <bool BF16, bool GATHER>
__global__ void __launch_bounds__(GATHER ? MlaPairTraits::THREADS_GATHER : MlaPairTraits::THREADS, 1)
    mla_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const DecodeParams p) {
  using T = MlaPairTraits;
  constexpr int NH = T::NH, NHC = T::NHC;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t cr = cluster_ctarank();  // 0: issues the pair UMMAs
  const uint32_t peer = cr ^ 1u;

  const int pair = blockIdx.x >> 1;
  const int hb = pair % p.head_blocks;
  const int rng = pair / p.head_blocks;
  const int nvalid = min(NH, p.G - hb * NH);

  const uint32_t ring = sbase + T::OFF_RING;
  const uint32_t qt = sbase + T::OFF_QT;
  const uint32_t pt = sbase + T::OFF_PT;
  float* red = reinterpret_cast<float*>(smem + T::OFF_RED);
  float* pmax_in = reinterpret_cast<float*>(smem + T::OFF_PMAX);
  float* m_sm = reinterpret_cast<float*>(smem + T::OFF_M);
  float* alpha_sm = reinterpret_cast<float*>(smem + T::OFF_ALPHA);
  float* l_sm = reinterpret_cast<float*>(smem + T::OFF_L);
  float* lpeer = reinterpret_cast<float*>(smem + T::OFF_LPEER);
  long long* scan = reinterpret_cast<long long*>(smem + T::OFF_SCAN);
  int* sched = reinterpret_cast<int*>(smem + T::OFF_SCHED);
  long long* pos = reinterpret_cast<long long*>(smem + T::OFF_POS);
  volatile int* merge_flag = reinterpret_cast<volatile int*>(smem + T::OFF_MERGE);
  volatile int* flags = reinterpret_cast<volatile int*>(smem + T::OFF_FLAGS);
  volatile int* abort_flag = flags + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + T::OFF_FLAGS + 12);
  const uint32_t bar0 = sbase + T::OFF_BAR;
  auto full_bar = [&](int g) { return bar0 + 8u * g; };
  auto empty_bar = [&](int g) { return bar0 + 8u * (T::RING_G + g); };
  const uint32_t q_full = bar0 + 8u * (2 * T::RING_G);
  const uint32_t q_free = q_full + 8;
  const uint32_t s_full = q_free + 8;        // [2]
  const uint32_t s_free = s_full + 16;       // [2] (CTA 0: both CTAs' softmax warps)
  const uint32_t p_local = s_free + 16;      // this CTA's own P^T rows written
  const uint32_t p_recv = p_local + 8;       // the other CTA's P^T rows landed (st.async bytes)
  const uint32_t p_peer = p_recv + 8;        // CTA 0: CTA 1's P^T buffer complete
  const uint32_t o_done = p_peer + 8;
  const uint32_t red_full = o_done + 8;      // [2]
  const uint32_t stat_ready = red_full + 16; // [2]
  const uint32_t xmax_full = stat_ready + 16;  // [2] peer maxima landed
  const uint32_t lsum_full = xmax_full + 16;   // peer sums landed
  const uint32_t drain = lsum_full + 8;
  const uint32_t mg_done = drain + 8;     // in-kernel merge: the softmax warps' stores fenced
  const uint32_t mg_flag = mg_done + 8;   // in-kernel merge: this CTA completed its unit half

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int g = 0; g < T::RING_G; ++g) {
      // top-k mode: one arrival per copying thread (when its copies have
      // landed), plus CTA 1's forwarded arrival on CTA 0's barrier
      mbar_init(full_bar(g), GATHER ? T::GATHER_THREADS + (cr == 0 ? 1 : 0) : 1);
      mbar_init(empty_bar(g), 1);
    }
    mbar_init(q_full, 1);
    mbar_init(q_free, 1);
    constexpr int SW = T::SOFTMAX_THREADS / 32;  // softmax warps
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full + 8 * i, 1);
      mbar_init(s_free + 8 * i, 2 * SW);      // one arrival per softmax warp of each CTA
      mbar_init(red_full + 8 * i, SW);
      mbar_init(stat_ready + 8 * i, NH / 32);
      mbar_init(xmax_full + 8 * i, 1);        // the local arm; the peer's bytes complete it
    }
    mbar_init(p_local, SW / 2);               // the warps writing this CTA's own heads
    mbar_init(p_recv, 1);
    mbar_init(p_peer, 1);
    mbar_init(o_done, 1);
    mbar_init(lsum_full, 1);
    mbar_init(drain, 1);
    mbar_init(mg_done, T::SOFTMAX_THREADS / 32);
    mbar_init(mg_flag, 1);
    flags[0] = 0;
    flags[1] = 0;
    flags[2] = 0;
    fence_mbar_init();  // release at cluster scope
    // the first tile's P^T rows from the other CTA (later tiles are armed by
    // the thread that sees the previous phase complete)
    mbar_arrive_expect_tx(p_recv, T::PT_PEER_BYTES);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), 512);
    tmem_relinquish_pair();
  }
  if (threadIdx.x == 0) pdl_launch_dependents();  // the combine may be scheduled now
  locate_range(p.skv, p.B, p.Hkv, T::TILE_SHIFT, p.ranges, rng, scan, sched, pos);
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers and the pair's TMEM exist
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int count = sched[3];
  auto walker = [&]() {
    PieceWalker w;
    w.skv = p.skv;
    w.B = p.B;
    w.Hkv = p.Hkv;
    w.shift = T::TILE_SHIFT;
    w.b = sched[0];
    w.kvh = sched[1];
    w.off = sched[2];
    w.remaining = count;
    w.gpos = pos[0];
    return w;
  };

  if (count > 0) {
    if (GATHER && warp >= T::GATHER_WARP0) {
      // ------------------------------------------------ producer: gathered K/V groups
      // The same groups in the same order as the copy producer below, each
      // filled from the selected cache rows with 16-byte cp.async copies,
      // eight lanes per 128-byte row chunk (coalesced), into the
      // 128-byte-swizzled layout a TMA copy would produce.  Warp gw copies
      // rows 64 gw .. 64 gw + 63 of every group; each lane's copies of a group
      // complete one arrival on the group's barrier.  A tile's row positions
      // are read once, while the previous tile's groups are copied (within
      // a piece), and kept for its V groups.  In CTA 1 warp 10 also forwards each group's arrival to CTA 0
      // two groups later (CTA 0's pair MMAs read this CTA's half of the group;
      // a proxy fence first: the copies are generic-proxy writes, the MMA
      // reads through the async proxy).
      const int gw = warp - T::GATHER_WARP0;
      const int rsub = lane >> 3, unit = lane & 7;
      const bool fwd = cr == 1 && gw == 0;
      const uint32_t lead = mapa_shared(full_bar(0), 0);
      int grp = 0, fgrp = 0, pending = 0;
      uint32_t ph = 0, fph = 0;
      bool ok = true;
      auto forward_one = [&]() {
        if (!ok) return;
        ok = mbar_wait_warp(full_bar(fgrp), fph, abort_flag, p.timeout_ns, 64);
        if (!ok) return;
        fence_proxy_async_smem();
        __syncwarp();
        if (elect_one()) mbar_arrive_remote_cta(lead + 8 * fgrp);
        __syncwarp();
        if (++fgrp == T::RING_G) { fgrp = 0; fph ^= 1u; }
        --pending;
      };
      // positions of keys row0 + 128 h + 64 gw + 32 k + lane (-1: a zero row)
      auto load_pos = [&](int row0, int b, int (&pr)[2][2]) {
        const int nsel = p.skv[b];
        const int len = p.src_len[b];
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const int key = row0 + 128 * h + 64 * gw + 32 * k + lane;
            int q = -1;
            if (key >= 0 && key < nsel) {
              q = p.idx[(int64_t)b * p.idx_sb + key];
              if (q < 0 || q >= len) {
                atomicOr(&g_attn_error, 4u);
                q = -1;
              }
            }
            pr[h][k] = q;
          }
      };
      auto gather = [&](int c0, int nch, const int (&pr)[2], int b) {
        if (!ok) return;
        ok = mbar_wait_warp_cluster(empty_bar(grp), ph ^ 1u, abort_flag, p.timeout_ns, 63);
        if (!ok) return;
        const uint8_t* sb0 = p.src + (int64_t)b * p.src_sb * 2;
        const uint32_t gbase = ring + grp * T::GBYTES;
#pragma unroll 4
        for (int i = 0; i < 16; ++i) {
          const int rl = 4 * i + rsub;  // row within this warp's 64
          const int q = __shfl_sync(0xffffffffu, pr[rl >> 5], rl & 31);
          const int r = 64 * gw + rl;   // row within the group
          const uint8_t* srow = sb0 + (int64_t)(q < 0 ? 0 : q) * p.src_ss * 2 + unit * 16;
          for (int cc = 0; cc < nch; ++cc)
            cp_async16(gbase + cc * T::SLOT + r * 128 + ((unit ^ (r & 7)) << 4),
                       srow + (c0 + cc) * 128, q < 0 ? 0u : 16u);
        }
        cp_async_arrive_noinc(full_bar(grp));
        if (++grp == T::RING_G) { grp = 0; ph ^= 1u; }
        if (fwd && ++pending > 2) forward_one();
      };
      PieceWalker w = walker();
      int b, kvh, t0, n;
      int cur[2][2], nxt[2][2], prev[2][2], prev_b = 0;
      bool have_prev = false;
      auto gather_v = [&]() {
        for (int m = 0; m < 2; ++m)
          for (int h = 0; h < 2; ++h) gather(4 * m + 2 * (int)cr, 2, prev[h], prev_b);
      };
      while (ok && w.next(b, kvh, t0, n)) {
        // a partial last pair tile is the 256 selections ending at the last
        // one (earlier keys masked); keys before the first are zero rows
        const int last_win = p.skv[b] - 256;
        load_pos(min(t0 * 256, last_win), b, nxt);
        for (int i = 0; i < n && ok; ++i) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            cur[h][0] = nxt[h][0];
            cur[h][1] = nxt[h][1];
          }
          // the next tile's positions load while this tile's groups are copied
          if (i + 1 < n) load_pos(min((t0 + i + 1) * 256, last_win), b, nxt);
          if (i == 0 && have_prev) gather_v();
          for (int c = 0; c < T::KCH; c += 2) gather(c, min(2, T::KCH - c), cur[cr], b);
          if (i > 0) gather_v();
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            prev[h][0] = cur[h][0];
            prev[h][1] = cur[h][1];
          }
          prev_b = b;
          have_prev = true;
        }
      }
      if (have_prev) gather_v();
      while (ok && fwd && pending > 0) forward_one();
      if (!ok) *abort_flag = 1;
    } else if (!GATHER && warp == 0 && lane == 0) {
      // ------------------------------------------------ producer: K/V groups
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      // K rows stay in L2 until the pair reads their first 512 columns again
      // as V (a tile later); that V read is their last use.
      const uint64_t pol_k = l2_policy_evict_normal();
      const uint64_t pol_v = l2_policy_evict_first();
      int grp = 0;
      uint32_t ph = 0;
      bool ok = true;
      // two chunks starting at `ch` of rows [row, row + 128); the bytes of
      // both CTAs' copies into group `grp` are counted on CTA 0's barrier
      auto load = [&](const CUtensorMap* map, int ch, int row, int kvh, int b, uint64_t pol) {
        if (!ok) return;
        ok = mbar_wait_cluster(empty_bar(grp), ph ^ 1u, abort_flag, p.timeout_ns, 41);
        if (!ok) return;
        if (cr == 0) mbar_arrive_expect_tx(full_bar(grp), 2 * T::GBYTES);
        tma_load_5d_pair(ring + grp * T::GBYTES, map, mapa_shared(full_bar(grp), 0), 0, row, ch,
                         kvh, b, pol);
        if (++grp == T::RING_G) { grp = 0; ph ^= 1u; }
      };
      PieceWalker w = walker();
      int b, kvh, t0, n;
      int pv_row = 0, pv_kvh = 0, pv_b = 0;  // pair tile whose V is still to be loaded
      bool have_prev = false;
      // V block m of this CTA = chunks 4m + 2cr, +1, for the tile's 256 keys
      auto load_v = [&]() {
        for (int m = 0; m < 2; ++m)
          for (int h = 0; h < 2; ++h)
            load(&tmV, 4 * m + 2 * (int)cr, pv_row + 128 * h, pv_kvh, pv_b, pol_v);
      };
      while (ok && w.next(b, kvh, t0, n)) {
        // a partial last pair tile is read as the 256 rows ending at the
        // sequence's last key (earlier rows masked), so no row past skv --
        // possibly unwritten memory -- is read; a negative start reads zeros
        const int last_win = p.skv[b] - 256;
        for (int i = 0; i < n && ok; ++i) {
          const int row0 = min((t0 + i) * 256, last_win);
          if (i == 0 && have_prev) load_v();  // finish the previous piece first
          for (int c = 0; c < T::KCH; c += 2) load(&tmK, c, row0 + 128 * (int)cr, kvh, b, pol_k);
          if (i > 0) load_v();
          pv_row = row0;
          pv_kvh = kvh;
          pv_b = b;
          have_prev = true;
        }
      }
      if (have_prev) load_v();
    } else if (warp == 0 && lane == 1) {
      // ------------------------------------------------ producer: Q^T half per piece
      tma_prefetch_desc(&tmQ);
      const uint64_t pol = l2_policy_evict_first();
      PieceWalker w = walker();
      int b, kvh, t0, n, k = 0;
      bool ok = true;
      while (ok && w.next(b, kvh, t0, n)) {
        if (k > 0)  // the previous piece's S^T MMAs have read the buffer
          ok = mbar_wait_cluster(q_free, (k - 1) & 1, abort_flag, p.timeout_ns, 42);
        if (!ok) break;
        if (cr == 0) mbar_arrive_expect_tx(q_full, 2 * T::QT_BYTES);
        const uint32_t lead = mapa_shared(q_full, 0);
        for (int c = 0; c < T::KCH; ++c)
          tma_load_3d_pair(qt + c * T::QT_CHUNK, &tmQ, lead, c * 64,
                           kvh * p.G + hb * NH + (int)cr * NHC, b, pol);
        ++k;
      }
    } else if (warp == 1 && cr == 0) {
      // ------------------------------------------------ pair MMA issuer
      constexpr uint32_t idS = umma_idesc(256, NH, BF16, false, false);
      constexpr uint32_t idO = umma_idesc(256, NH, BF16, true, true);
      int grp = 0;
      uint32_t ph = 0;
      bool ok = true;
      auto pv = [&](int t, bool first_of_piece) {
        if (!ok) return;
        // P^T of tile t complete in both CTAs: this CTA's own rows, the rows
        // CTA 1 sent here, and CTA 1's buffer (forwarded by CTA 1)
        ok = mbar_wait_warp(p_local, t & 1, abort_flag, p.timeout_ns, 43) &&
             mbar_wait_warp_cluster(p_recv, t & 1, abort_flag, p.timeout_ns, 48) &&
             mbar_wait_warp_cluster(p_peer, t & 1, abort_flag, p.timeout_ns, 49);
        if (!ok) return;
        if (elect_one()) mbar_arrive_expect_tx(p_recv, T::PT_PEER_BYTES);  // next tile's rows
        __syncwarp();
        fence_proxy_async_smem();  // the st.async rows, for the MMA's operand reads
        tc_fence_after();
        for (int m = 0; m < 2; ++m) {
          for (int h = 0; h < 2; ++h) {
            ok = mbar_wait_warp_cluster(full_bar(grp), ph, abort_flag, p.timeout_ns, 44);
            if (!ok) return;
            tc_fence_after();
            if constexpr (GATHER) fence_proxy_async_smem();  // this CTA's cp.async rows
            if (elect_one()) {
              // A = V^T (MN-major, 128-byte swizzle): the group's two chunks are
              // the block's two 64-row halves (LBO = one chunk), 8-key groups
              // 1024 bytes apart, 16 keys per K step = 2048 bytes.
              const uint64_t ad0 = umma_sdesc(ring + grp * T::GBYTES, T::SLOT, 1024, SMEM_SW128);
              // B = P^T (MN-major, no swizzle): keys 128h.. of the pair tile;
              // 8-key groups NHC*16 = 1024 bytes apart (LBO), 8-head groups
              // 128 bytes apart (SBO).
              const uint64_t bd0 = umma_sdesc(pt + h * (T::TILE / 8) * NHC * 16, NHC * 16, 128,
                                              SMEM_NOSWIZZLE);
              const uint32_t d = tmem + T::TMEM_O + m * 128;
              umma_ss_pair(d, ad0, bd0, idO, (first_of_piece && h == 0) ? 0u : 1u);
#pragma unroll
              for (int ks = 1; ks < 8; ++ks)
                umma_ss_pair(d, ad0 + (uint64_t)(ks * (2048 >> 4)),
                             bd0 + (uint64_t)(ks * (2 * NHC * 16 >> 4)), idO, 1u);
              umma_commit_pair(empty_bar(grp));
            }
            __syncwarp();
            if (++grp == T::RING_G) { grp = 0; ph ^= 1u; }
          }
        }
        if (elect_one()) umma_commit_pair(o_done);
        __syncwarp();
      };
      PieceWalker w = walker();
      int b, kvh, t0, n, j = 0, k = 0;
      bool prev_first = false;
      while (ok && w.next(b, kvh, t0, n)) {
        for (int i = 0; i < n && ok; ++i, ++j) {
          const int sb = j & 1;
          if (i == 0 && j > 0) pv(j - 1, prev_first);  // finish the previous piece first
          if (i == 0) {
            ok = ok && mbar_wait_warp_cluster(q_full, k & 1, abort_flag, p.timeout_ns, 45);
            if (!ok) break;
            tc_fence_after();
          }
          if (j >= 2)  // both CTAs' softmax has read S^T(j - 2)
            ok = mbar_wait_warp_cluster(s_free + 8 * sb, ((j >> 1) - 1) & 1, abort_flag,
                                        p.timeout_ns, 46);
          if (!ok) break;
          tc_fence_after();
          for (int c = 0; c < T::KCH && ok; c += 2) {
            ok = mbar_wait_warp_cluster(full_bar(grp), ph, abort_flag, p.timeout_ns, 47);
            if (!ok) break;
            tc_fence_after();
            if constexpr (GATHER) fence_proxy_async_smem();  // this CTA's cp.async rows
            if (elect_one()) {
              // A = K rows (each CTA its own 128 keys), B = Q^T chunks (each CTA
              // its 64 heads): K-major, 128-byte swizzle, 32 bytes per K step.
              const uint64_t ad0 = umma_sdesc(ring + grp * T::GBYTES, 16, 1024, SMEM_SW128);
              const uint64_t bd0 = umma_sdesc(qt + c * T::QT_CHUNK, 16, 1024, SMEM_SW128);
              const uint32_t d = tmem + T::TMEM_S + sb * NH;
              umma_ss_pair(d, ad0, bd0, idS, c > 0 ? 1u : 0u);
#pragma unroll
              for (int ks = 1; ks < 4; ++ks) umma_ss_pair(d, ad0 + 2 * ks, bd0 + 2 * ks, idS, 1u);
              if (c + 1 < T::KCH) {
                const uint64_t ad1 = ad0 + (T::SLOT >> 4);
                const uint64_t bd1 = bd0 + (T::QT_CHUNK >> 4);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) umma_ss_pair(d, ad1 + 2 * ks, bd1 + 2 * ks, idS, 1u);
              }
              umma_commit_pair(empty_bar(grp));
            }
            __syncwarp();
            if (++grp == T::RING_G) { grp = 0; ph ^= 1u; }
          }
          if (!ok) break;
          if (elect_one()) {
            umma_commit_pair(s_full + 8 * sb);
            if (i == n - 1) umma_commit_pair(q_free);
          }
          __syncwarp();
          if (i > 0) pv(j - 1, prev_first);
          prev_first = (i == 0);
        }
        ++k;
      }
      if (ok && j > 0) pv(j - 1, prev_first);
    } else if (warp == 1) {
      // ------------------------------------------------ CTA 1: P^T forwarder
      // CTA 0's MMAs read this CTA's P^T buffer: once this CTA's own rows are
      // written and the rows from CTA 0 have landed, tell CTA 0.
      const uint32_t p_peer_lead = mapa_shared(p_peer, 0);
      PieceWalker w = walker();
      int b, kvh, t0, n, j = 0;
      bool ok = true;
      while (ok && w.next(b, kvh, t0, n)) {
        for (int i = 0; i < n && ok; ++i, ++j) {
          ok = mbar_wait_warp(p_local, j & 1, abort_flag, p.timeout_ns, 61) &&
               mbar_wait_warp_cluster(p_recv, j & 1, abort_flag, p.timeout_ns, 62);
          if (!ok) break;
          if (elect_one()) mbar_arrive_expect_tx(p_recv, T::PT_PEER_BYTES);
          __syncwarp();
          fence_proxy_async_smem();
          __syncwarp();
          if (elect_one()) mbar_arrive_remote_cta(p_peer_lead);
          __syncwarp();
        }
      }
    } else if (warp >= 2 && warp < T::GATHER_WARP0) {
      // ------------------------------------------------ softmax + epilogues
      constexpr int HH = NHC;                  // heads per thread (64)
      const int st = threadIdx.x - 64;         // 0..255
      const int half = st >> 7;                // heads [64 half, 64 half + 64)
      const int h0l = half * HH;
      const int wq = warp & 3;
      const int row = wq * 32 + lane;          // key row of S^T / d row of O^T blocks
      const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
      volatile int own_abort = 0;
      // barriers completed by the other CTA (arrivals, st.async bytes, pair
      // commits) are waited on with cluster-scope acquire, local ones at CTA scope
      auto wait = [&](uint32_t bar, uint32_t parity, uint32_t id) {
        return mbar_wait_warp_cluster(bar, parity, &own_abort, p.timeout_ns, id);
      };
      auto wait_l = [&](uint32_t bar, uint32_t parity, uint32_t id) {
        return mbar_wait_warp(bar, parity, &own_abort, p.timeout_ns, id);
      };
      // where this thread's P^T row goes: its heads are CTA `half`'s columns;
      // rows for the other CTA go by st.async, counted on that CTA's p_recv
      const bool local_heads = half == (int)cr;
      const uint32_t pdst = local_heads ? pt : mapa_shared(pt, (uint32_t)half);
      const uint32_t p_recv_peer = mapa_shared(p_recv, peer);
      const uint32_t s_free_lead = mapa_shared(s_free, 0);
      if (st < NH) m_sm[st] = -INFINITY;
      named_bar_sync(1, T::SOFTMAX_THREADS);

      PieceWalker w = walker();
      int b, kvh, t0, n, j = 0, r = 0, pc = 0;
      long long gstart;
      bool ok = true;
      while (ok && w.next(b, kvh, t0, n, gstart)) {
        const int skv_b = p.skv[b];
        const int64_t slot_id = (int64_t)rng + (int64_t)b * p.Hkv + kvh;
        float l[HH];
#pragma unroll
        for (int h = 0; h < HH; ++h) l[h] = 0.f;

        for (int i = 0; i < n && ok; ++i, ++j, ++r) {
          const int sb = j & 1;
          const int rb = r & 1;
          const uint32_t rpar = (r >> 1) & 1;
          ok = wait(s_full + 8 * sb, (j >> 1) & 1, 51);
          if (!ok) break;
          tc_fence_after();
          // rows of a partial last tile end at skv_b; those before the
          // tile's start belong to the previous tile
          const int tile0 = (t0 + i) * 256;
          const bool valid = min(tile0, skv_b - 256) + (int)cr * T::TILE + row >= tile0;
          const uint32_t s_col = tmem + lane_base + T::TMEM_S + sb * NH + h0l;

          // this CTA's per-head maximum over its 128 keys
          float* rbuf = red + rb * 4 * NH;
          {
            float v[HH];
            tmem_ld<HH>(s_col, v);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < HH; ++e) v[e] = valid ? v[e] * p.scale_log2 : -INFINITY;
            transposed_warp_max<HH, HH, 16>(v, lane);
#pragma unroll
            for (int e = 0; e < HH / 32; ++e) rbuf[wq * NH + h0l + transposed_head<HH>(lane, e)] = v[e];
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(red_full + 8 * rb);
          ok = wait_l(red_full + 8 * rb, rpar, 52);
          if (!ok) break;
          if (st == 0) flags[rb ^ 1] = 0;
          if (st < NH) {
            // swap tile maxima with the other CTA; both then hold the same
            // maximum over the pair tile's 256 keys
            const float own =
                fmaxf(fmaxf(rbuf[st], rbuf[NH + st]), fmaxf(rbuf[2 * NH + st], rbuf[3 * NH + st]));
            st_async_f32(mapa_shared(smem_u32(pmax_in + (j & 1) * NH + st), peer), own,
                         mapa_shared(xmax_full + 8 * (j & 1), peer));
            if (st == 0) mbar_arrive_expect_tx(xmax_full + 8 * (j & 1), NH * 4);  // the peer's maxima
            ok = wait(xmax_full + 8 * (j & 1), (j >> 1) & 1, 53);
            if (ok) {
              const float tm = fmaxf(own, pmax_in[(j & 1) * NH + st]);
              const float mo = m_sm[st];
              // lazy raise (threshold 8 in log2 units), as in the one-SM kernel
              const bool need = tm > mo + 8.f;
              const float mn = need ? tm : mo;
              alpha_sm[st] = need ? ex2(mo - mn) : 1.f;
              m_sm[st] = mn;
              if (need) flags[rb] = 1;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(stat_ready + 8 * rb);
          }
          if (!ok) break;
          ok = wait_l(stat_ready + 8 * rb, rpar, 54);
          if (!ok) break;
          const bool any = flags[rb] != 0;

          // P^T buffer: PV(j - 1) must be done (single buffer, both CTAs write it)
          if (j >= 1) {
            ok = wait(o_done, (j - 1) & 1, 55);
            if (!ok) break;
            tc_fence_after();
          }
          if (any && i > 0) {  // rescale this thread's O^T columns
#pragma unroll 1
            for (int m = 0; m < 2; ++m) {
#pragma unroll 1
              for (int c0 = 0; c0 < HH; c0 += 16) {
                float o[16];
                const uint32_t ta = tmem + lane_base + T::TMEM_O + m * 128 + h0l + c0;
                tmem_ld16(ta, o);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 16; c += 4) {
                  const float4 a4 = *reinterpret_cast<const float4*>(alpha_sm + h0l + c0 + c);
                  o[c] *= a4.x;
                  o[c + 1] *= a4.y;
                  o[c + 2] *= a4.z;
                  o[c + 3] *= a4.w;
                }
                tmem_st16(ta, o);
              }
            }
            tmem_wait_st();
          }
          if (any) {
#pragma unroll
            for (int h = 0; h < HH; h += 4) {
              const float4 a4 = *reinterpret_cast<const float4*>(alpha_sm + h0l + h);
              l[h] *= a4.x;
              l[h + 1] *= a4.y;
              l[h + 2] *= a4.z;
              l[h + 3] *= a4.w;
            }
          }

          // weights: S^T read again in 16-column pieces; P^T row of key
          // 128 cr + row for this thread's 64 heads, as 8 core-matrix rows
          const int kk = (int)cr * T::TILE + row;
          const uint32_t prow = pdst + (kk >> 3) * (NHC * 16) + (kk & 7) * 16;
#pragma unroll
          for (int c0 = 0; c0 < HH; c0 += 16) {
            float sv[16];
            tmem_ld16(s_col + c0, sv);
            tmem_wait_ld();
            uint32_t u[8];
#pragma unroll
            for (int e = 0; e < 16; e += 4) {
              const float4 m4 = *reinterpret_cast<const float4*>(m_sm + h0l + c0 + e);
              const float mm[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
              for (int q = 0; q < 4; q += 2) {
                // an invalid row's weights are exactly 0 (ex2(-inf) = +0)
                const float p0 = valid ? ex2(fmaf(sv[e + q], p.scale_log2, -mm[q])) : 0.f;
                const float p1 = valid ? ex2(fmaf(sv[e + q + 1], p.scale_log2, -mm[q + 1])) : 0.f;
                u[(e + q) >> 1] = pack2(p0, p1, BF16);
                l[c0 + e + q] += p0;
                l[c0 + e + q + 1] += p1;
              }
            }
            const uint32_t a0 = prow + ((c0 >> 3) + 0) * 128;
            const uint32_t a1 = prow + ((c0 >> 3) + 1) * 128;
            if (local_heads) {
              st_shared_v4(a0, u[0], u[1], u[2], u[3]);
              st_shared_v4(a1, u[4], u[5], u[6], u[7]);
            } else {
              st_async_v4(a0, u[0], u[1], u[2], u[3], p_recv_peer);
              st_async_v4(a1, u[4], u[5], u[6], u[7], p_recv_peer);
            }
          }
          // S^T(j) has been read (a signal without data: CTA 1 arrives relaxed)
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if (cr == 0) mbar_arrive(s_free + 8 * sb);
            else mbar_arrive_remote_relaxed(s_free_lead + 8 * sb);
          }
          if (local_heads) {  // this CTA's own P^T rows, for the MMA's operand reads
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_local);
          }
        }
        if (!ok) break;

        // ---------------------------------------------- epilogue of the piece
        {
          const int t = j - 1;
          ok = wait(o_done, t & 1, 56);
          if (!ok) break;
          tc_fence_after();
          const int rb = r & 1;
          const uint32_t rpar = (r >> 1) & 1;
          float* rbuf = red + rb * 4 * NH;
          transposed_warp_sum<HH, HH, 16>(l, lane);
#pragma unroll
          for (int e = 0; e < HH / 32; ++e) rbuf[wq * NH + h0l + transposed_head<HH>(lane, e)] = l[e];
          __syncwarp();
          if (lane == 0) mbar_arrive(red_full + 8 * rb);
          ok = wait_l(red_full + 8 * rb, rpar, 57);
          if (!ok) break;
          if (st == 0) flags[rb ^ 1] = 0;
          if (st < NH) {
            const float own = (rbuf[st] + rbuf[NH + st]) + (rbuf[2 * NH + st] + rbuf[3 * NH + st]);
            st_async_f32(mapa_shared(smem_u32(lpeer + st), peer), own, mapa_shared(lsum_full, peer));
            if (st == 0) mbar_arrive_expect_tx(lsum_full, NH * 4);  // the peer's sums
            ok = wait(lsum_full, pc & 1, 58);
            if (ok) {
              // the same sum in both CTAs: CTA 0's keys first
              const float L = cr == 0 ? own + lpeer[st] : lpeer[st] + own;
              l_sm[st] = L;
              // both CTAs write the (identical) LSE: the merge of either
              // half of the output reads it
              if (st < nvalid)
                p.ws_lse[slot_id * p.G + hb * NH + st] =
                    L > 0.f ? (m_sm[st] + __log2f(L)) * 0.69314718055994531f : -INFINITY;
              m_sm[st] = -INFINITY;  // the next piece starts afresh
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(stat_ready + 8 * rb);
          }
          if (!ok) break;
          ok = wait_l(stat_ready + 8 * rb, rpar, 59);
          if (!ok) break;
          ++r;
          ++pc;
#pragma unroll 1
          for (int m = 0; m < 2; ++m) {
            const int dd = 256 * m + (int)cr * 128 + row;  // this thread's O^T row = d
#pragma unroll 1
            for (int c0 = 0; c0 < HH; c0 += 16) {
              float o[16];
              tmem_ld16(tmem + lane_base + T::TMEM_O + m * 128 + h0l + c0, o);
              tmem_wait_ld();
#pragma unroll
              for (int c = 0; c < 16; ++c) {
                const int h = h0l + c0 + c;
                if (h < nvalid) {
                  const float L = l_sm[h];
                  p.ws_o[(slot_id * p.G + hb * NH + h) * T::DV + dd] = L > 0.f ? o[c] / L : 0.f;
                }
              }
            }
          }
          tc_fence_before();
          // the CTA that completes its half (d rows) of the unit's key tiles
          // merges that half of the unit's pieces into the output
          if (p.counters) {
            const int unit = b * p.Hkv + kvh;
            const int tb = key_tiles(skv_b, T::TILE_SHIFT);
            const bool last = arrive_last(
                p.counters + ((int64_t)unit * p.head_blocks + hb) * 2 + cr, n, tb, mg_done,
                mg_flag, (pc - 1) & 1, warp == 2, merge_flag, &own_abort, p.timeout_ns);
            if (last) {
              long long slot0;
              const int np = unit_pieces(gstart, t0, tb, unit, pos, slot0);
              constexpr int TPC = T::SOFTMAX_THREADS / NH;  // threads per head
              for (int m = 0; m < 2; ++m)  // d rows 256 m + 128 cr .. + 127
                merge_unit<BF16, TPC, 128 / 4 / TPC>(p, T::DV, p.G, slot0, np, b, kvh, hb * NH,
                                                     nvalid, 256 * m + 128 * (int)cr,
                                                     cr == 0 && m == 0, st);
            }
          }
        }
      }
      if (!ok) *abort_flag = 1;
    }
  }

  // Common exit.  After a give-up in either CTA, CTA 0's issued UMMAs (which
  // read both CTAs' shared memory and write both TMEMs) and every CTA's
  // issued copies must land before the pair leaves.
  __syncthreads();
  if (*abort_flag) {
    if (warp == 1 && cr == 0) {
      if (elect_one()) umma_commit_pair(drain);
      __syncwarp();
      volatile int never = 0;
      mbar_wait_warp(drain, 0, &never, 1000000ull, 60);
    }
    if (threadIdx.x == 0) {
      const uint64_t t0n = global_timer_ns();
      while (global_timer_ns() - t0n < 2000000ull) __nanosleep(1000);
    }
  }
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace attn
