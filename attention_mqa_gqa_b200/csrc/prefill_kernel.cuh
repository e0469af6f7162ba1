// prefill_kernel.cuh -- causal (or full) attention forward for Sq > 1.
//
// Prefill is the quadratic phase ("GQA和MLA详解" section 1: T enters both
// matmuls as M and N) and is compute-bound, so both matmuls run on the
// tensor cores.  The T x T score matrix is never materialised: keys are
// streamed in tiles of 128 with an online softmax ("带你了解Attention"
// section 6.3, FlashAttention: tiling plus online softmax; "GQA和MLA详解"
// section 4, shared-memory tiling).
//
// One work item is 128 query rows of one head and DVH output columns:
//
//   S[128 x 128]   = Q_tile[128 x d_k] * K_tile^T            (tcgen05 -> TMEM)
//   P = exp2(S*scale*log2e - m), row max m kept per thread (thread = row)
//   O[128 x DVH]  += P[128 x 128] * V_tile[128 x DVH]        (tcgen05, A from TMEM)
//
// P (bf16) is written back into the first 64 columns of its own S buffer
// and read from there by the PV MMA, so it takes no shared memory and no
// shared-memory bandwidth; the S buffer is reused for tile j + 2 once PV(j)
// has completed.
//
// TMEM holds 512 fp32 columns per SM: two S buffers (256 columns) and O
// (DVH = 128 columns).  (At d_k = d_v = 512 a 128 x 512 fp32 O alone fills
// TMEM; that case runs on SM pairs that split the two matmuls, in
// prefill_ab_kernel.cuh.)
//
// The grid is persistent: one CTA per SM walks the work items in
// heavy-first order (the last q tiles see the most keys under the causal
// mask) with a stride of the grid size, so the next item's Q load and K/V
// stream overlap the current item's last MMAs and epilogue.
//
// Warp roles: warp 0 lane 0 streams K/V chunks through a ring of 32 KB
// groups and lane 1 loads Q per item (TMA), warp 1 allocates TMEM and issues
// UMMA, the other 16 warps run the softmax, rescale and epilogue: SPLIT
// threads per q row (warps with the same index mod 4
// share a TMEM lane quarter), each owning a slice of the row's keys and of
// its output columns, exchanging the row maximum and sum through shared
// memory.
#pragma once

#include "sm100.cuh"

namespace attn {

struct PrefillParams {
  void* out;                  // [B, Hq, Sq, d_v]
  int64_t o_sb, o_sh, o_ss;   // element strides of out
  float* lse;                 // [B, Hq, Sq] or NULL
  const int32_t* skv;         // [B] (device)
  int B, Hq, Hkv, G, Sq;
  int n_qtiles, dv_parts, n_items;
  int heads_per_block;        // q heads (a multiple of G) whose items run together
  float scale_log2;           // scale * log2(e), scale > 0
  int causal;
  uint64_t timeout_ns;
};

struct PrefillItem {
  int part, h, b, kvh, q0, skv, ntiles;
};

// Work item L.  The q heads are taken in blocks of heads_per_block whose
// K/V together fit comfortably in L2 (the items of one block run at about
// the same time, so each K/V tile comes from DRAM about once); inside a
// block the heaviest q tiles come first, and the dv parts and heads of one
// q tile are adjacent so that CTAs running at the same time read the same
// K/V tiles.
__device__ __forceinline__ PrefillItem prefill_item(const PrefillParams& p, int L) {
  PrefillItem it;
  const int units = p.Hq, units_per_block = p.heads_per_block;
  const int per_head = p.n_qtiles * p.B * p.dv_parts;
  const int blk = L / (units_per_block * per_head);
  L -= blk * units_per_block * per_head;
  const int h0 = blk * units_per_block;
  const int nh = min(units_per_block, units - h0);  // head units of this block
  it.part = L % p.dv_parts;
  L /= p.dv_parts;
  it.h = h0 + L % nh;
  L /= nh;
  it.b = L % p.B;
  const int qt = p.n_qtiles - 1 - L / p.B;
  it.kvh = it.h / p.G;
  it.q0 = qt * 128;
  it.skv = p.skv[it.b];
  const int q_last = min(it.q0 + 127, p.Sq - 1);
  int lim_last = p.causal ? q_last + it.skv - p.Sq + 1 : it.skv;  // keys the last row sees
  lim_last = max(0, min(it.skv, lim_last));
  it.ntiles = (lim_last + 127) / 128;
  return it;
}

template <int DK, int DVH>
struct PrefillTraits {
  static constexpr int TILE = 128;               // q rows per item (MMA M)
  static constexpr int KT = 128;                 // keys per tile (MMA N of S)
  static constexpr int KCH = DK / 64;            // 64-column chunks of a Q / K row
  static constexpr int QCH = (KCH + 1) & ~1;     // chunk slots per Q row: pairs, the
                                                 // last one zero-filled if KCH is odd
  static constexpr int VCH = DVH / 64;           // V chunks per key tile (this item's columns)
  // softmax threads per q row: 4 (the softmax is bound by instruction
  // issue: more warps hide more latency)
  static constexpr int SPLIT = 4;
  static constexpr int NQ = QCH > 2 ? 1 : 2;     // Q buffers
  static constexpr int RING = 8;                 // 16 KB chunk slots
  static constexpr int SLOT = 16384;
  // one TMA copy moves GCH consecutive 64-column chunks (one ring group):
  // copies of a single 16 KB chunk cap a CTA's stream well below what the
  // tensor cores consume
  static constexpr int GCH = 2;
  static constexpr int GBYTES = GCH * SLOT;
  static constexpr int RING_G = RING / GCH;
  static constexpr int Q_BYTES = QCH * SLOT;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_RING = OFF_Q + NQ * Q_BYTES;
  // row exchange buffers float [XR][SPLIT][128]: two rounds alternate with
  // the tile (one barrier per exchange)
  static constexpr int XR = 2;
  static constexpr int OFF_XCH = OFF_RING + RING * SLOT;
  static constexpr int OFF_FLAGS = OFF_XCH + XR * SPLIT * 128 * 4;  // abort, tmem base
  static constexpr int OFF_BAR = OFF_FLAGS + 16;
  // full[RING_G], empty[RING_G], q_full[NQ], q_free[NQ], s_full[2], p_full[2],
  // o_done[2] (one of each per S/P buffer), o_free, drain
  static constexpr int NBAR = 2 * RING_G + 2 * NQ + 8;
  static constexpr int SOFTMAX_THREADS = 128 * SPLIT;
  static constexpr int THREADS = 64 + SOFTMAX_THREADS;
  static constexpr int SMEM_BYTES = OFF_BAR + NBAR * 8 + 1024;
  static constexpr int TMEM_S = 0;               // two S buffers, 128 columns each; P(j)
                                                 // overwrites the first 64 of S(j)
  static constexpr int TMEM_O = 256;             // DVH columns
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(VCH % GCH == 0 && QCH % GCH == 0 && RING % GCH == 0 && GCH == 2,
                "chunks travel in pairs; a V pair is one 128-column block of O");
  static_assert(TMEM_O + DVH <= 512, "TMEM");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

template <int DK, int DVH, bool BF16>
__global__ void __launch_bounds__(PrefillTraits<DK, DVH>::THREADS, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
  using T = PrefillTraits<DK, DVH>;
  const int item0 = (int)blockIdx.x;
  const int istride = (int)gridDim.x;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);

  const uint32_t qs = sbase + T::OFF_Q;
  const uint32_t ring = sbase + T::OFF_RING;
  float* xch = reinterpret_cast<float*>(smem + T::OFF_XCH);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + T::OFF_FLAGS);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + T::OFF_FLAGS + 4);
  const uint32_t bar0 = sbase + T::OFF_BAR;
  auto full_bar = [&](int g) { return bar0 + 8u * g; };
  auto empty_bar = [&](int g) { return bar0 + 8u * (T::RING_G + g); };
  const uint32_t q_full = bar0 + 8u * (2 * T::RING_G);  // [NQ]
  const uint32_t q_free = q_full + 8 * T::NQ;          // [NQ]
  const uint32_t s_full = q_free + 8 * T::NQ;          // [2] S(j) in buffer j & 1
  const uint32_t p_full = s_full + 16;                 // [2] P(j) written over S(j)
  const uint32_t o_done = p_full + 16;                 // [2] PV(j) completed
  const uint32_t o_free = o_done + 16;
  const uint32_t drain = o_free + 8;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int g = 0; g < T::RING_G; ++g) {
      mbar_init(full_bar(g), 1);
      mbar_init(empty_bar(g), 1);
    }
    for (int i = 0; i < T::NQ; ++i) {
      mbar_init(q_full + 8 * i, 1);
      mbar_init(q_free + 8 * i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full + 8 * i, 1);
      mbar_init(p_full + 8 * i, T::SOFTMAX_THREADS);
      mbar_init(o_done + 8 * i, 1);
    }
    mbar_init(o_free, T::SOFTMAX_THREADS);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), T::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  auto wait1 = [&](uint32_t bar, uint32_t parity, volatile int* ab, uint32_t id) {
    return mbar_wait(bar, parity, ab, p.timeout_ns, id);
  };
  auto waitw = [&](uint32_t bar, uint32_t parity, volatile int* ab, uint32_t id) {
    return mbar_wait_warp(bar, parity, ab, p.timeout_ns, id);
  };

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------- producer: K/V ring
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    const uint64_t pol_kv = l2_policy_evict_last();  // shared by the group's heads
    int grp = 0;
    uint32_t ph = 0;
    bool ok = true;
    // one copy (32 KB) of chunks [ch, ch + GCH) of key rows [row, row +
    // 128) -> the next ring group
    auto load = [&](const CUtensorMap* map, int ch, int row, int kvh, int b) {
      if (!ok) return;
      ok = wait1(empty_bar(grp), ph ^ 1u, abort_flag, 21);
      if (!ok) return;
      mbar_arrive_expect_tx(full_bar(grp), T::GBYTES);
      tma_load_5d(ring + grp * T::GBYTES, map, full_bar(grp), 0, row, ch, kvh, b, pol_kv);
      if (++grp == T::RING_G) { grp = 0; ph ^= 1u; }
    };
    bool have_prev = false;
    int pv_tok = 0, pv_kvh = 0, pv_b = 0, pv_ch = 0;  // tile whose V is still to load
    // A partial last key tile is read as the KT rows ending at the
    // sequence's last key (the rows before the tile are masked), so no row
    // past skv -- possibly unwritten memory -- enters P.V; a negative start
    // reads zeros.
    auto load_v = [&]() {
      for (int c = 0; c < T::VCH; c += T::GCH) load(&tmV, pv_ch + c, pv_tok, pv_kvh, pv_b);
    };
    for (int L = item0; L < p.n_items && ok; L += istride) {
      const PrefillItem it = prefill_item(p, L);
      for (int j = 0; j < it.ntiles && ok; ++j) {
        if (j == 0 && have_prev) load_v();  // finish the previous item first
        const int row0 = min(j * T::KT, it.skv - T::KT);
        for (int c = 0; c < T::KCH; c += T::GCH) load(&tmK, c, row0, it.kvh, it.b);
        if (j > 0) load_v();
        pv_tok = row0;
        pv_kvh = it.kvh;
        pv_b = it.b;
        pv_ch = it.part * (DVH / 64);
        have_prev = true;
      }
    }
    if (have_prev) load_v();
  } else if (warp == 0 && lane == 1) {
    // ---------------------------------------------------- producer: Q per item
    tma_prefetch_desc(&tmQ);
    const uint64_t pol_q = l2_policy_evict_first();
    int kq = 0;
    bool ok = true;
    for (int L = item0; L < p.n_items && ok; L += istride) {
      const PrefillItem it = prefill_item(p, L);
      if (it.ntiles == 0) continue;
      const int qb = kq % T::NQ;
      if (kq >= T::NQ)  // buffer qb was last read by the S MMAs of item kq - NQ
        ok = wait1(q_free + 8 * qb, ((kq - T::NQ) / T::NQ) & 1, abort_flag, 22);
      if (!ok) break;
      mbar_arrive_expect_tx(q_full + 8 * qb, T::Q_BYTES);
      for (int c = 0; c < T::QCH; c += T::GCH)
        tma_load_5d(qs + qb * T::Q_BYTES + c * T::SLOT, &tmQ, q_full + 8 * qb, 0, it.q0, c, it.h,
                    it.b, pol_q);
      ++kq;
    }
  } else if (warp == 1) {
    // ---------------------------------------------------- MMA issuer (whole warp,
    // one elected lane issues; waits are polled by the converged warp)
    constexpr uint32_t idS = umma_idesc(128, 128, BF16, false, false);  // Q, K both K-major
    constexpr uint32_t idO = umma_idesc(128, 128, BF16, false, true);   // P K, V MN-major
    auto mma_ss = [&](uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
      umma_ss(d, a, b, id, acc);
    };
    auto mma_ts = [&](uint32_t d, uint32_t a, uint64_t b, uint32_t id, uint32_t acc) {
      umma_ts(d, a, b, id, acc);
    };
    auto commit = [&](uint32_t bar) { umma_commit(bar); };
    int grp = 0;
    uint32_t ph = 0;
    bool ok = true;
    // PV(t): O += P(t) V(t); the first tile of item k > 0 first waits until
    // the epilogue of item k-1 has read O out of TMEM.
    auto pv = [&](int t, bool first, int k) {
      if (!ok) return;
      const int pb = t & 1;
      ok = waitw(p_full + 8 * pb, (t >> 1) & 1, abort_flag, 23);
      if (ok && first && k > 0) ok = waitw(o_free, (k - 1) & 1, abort_flag, 24);
      if (!ok) return;
      tc_fence_after();
      const uint32_t pcol = tmem + T::TMEM_S + pb * 128;  // P(t): 8 columns per 16 keys
      for (int i = 0; i < T::VCH / 2; ++i) {  // one ring group = 128 columns of V
        ok = waitw(full_bar(grp), ph, abort_flag, 25);
        if (!ok) return;
        tc_fence_after();
        const uint32_t bbase = ring + grp * T::GBYTES;
        if (elect_one()) {
          // B = V: MN-major (d contiguous), 128-byte swizzle; the two 64-column
          // halves are the group's two chunks (LBO), 8-key groups 1024 bytes
          // (SBO), 16 keys per K step = 2048 bytes.  A = P(t) from TMEM.
          const uint64_t bd0 = umma_sdesc(bbase, T::SLOT, 1024, SMEM_SW128);
          const uint32_t d = tmem + T::TMEM_O + i * 128;
          mma_ts(d, pcol, bd0, idO, first ? 0u : 1u);
#pragma unroll
          for (int ks = 1; ks < 8; ++ks)
            mma_ts(d, pcol + ks * 8, bd0 + (uint64_t)(ks * (2048 >> 4)), idO, 1u);
          commit(empty_bar(grp));
        }
        __syncwarp();
        if (++grp == T::RING_G) { grp = 0; ph ^= 1u; }
      }
      if (elect_one()) commit(o_done + 8 * pb);
      __syncwarp();
    };
    int j = 0, kq = 0, prev_k = 0;
    bool prev_first = false;
    for (int L = item0; L < p.n_items && ok; L += istride) {
      const PrefillItem it = prefill_item(p, L);
      if (it.ntiles == 0) continue;
      const int qb = kq % T::NQ;
      for (int i = 0; i < it.ntiles && ok; ++i, ++j) {
        const int sb = j & 1;
        if (i == 0 && j > 0) pv(j - 1, prev_first, prev_k);  // finish the previous item
        if (i == 0) {
          ok = ok && waitw(q_full + 8 * qb, (kq / T::NQ) & 1, abort_flag, 26);
          if (!ok) break;
        }
        // S buffer sb last held P(j - 2): PV(j - 2) must have completed
        if (j >= 2) ok = waitw(o_done + 8 * sb, ((j - 2) >> 1) & 1, abort_flag, 27);
        if (!ok) break;
        tc_fence_after();
        for (int c = 0; c < T::KCH && ok; c += T::GCH) {
          ok = waitw(full_bar(grp), ph, abort_flag, 28);
          if (!ok) break;
          tc_fence_after();
          if (elect_one()) {
            // A = Q chunks c.., B = the group's K chunks: both K-major, 128-byte
            // swizzle, 8-row groups 1024 bytes apart, 32 bytes per K step; a K
            // chunk of the group is 128 keys x 128 bytes.
            const uint64_t ad0 = umma_sdesc(qs + qb * T::Q_BYTES + c * T::SLOT, 16, 1024, SMEM_SW128);
            const uint64_t bd0 = umma_sdesc(ring + grp * T::GBYTES, 16, 1024, SMEM_SW128);
            const uint32_t d = tmem + T::TMEM_S + sb * 128;
            mma_ss(d, ad0, bd0, idS, c > 0 ? 1u : 0u);
            // the second chunk of an odd count's last pair is padding: skipped
            const int nks = c + T::GCH <= T::KCH ? 4 * T::GCH : 4 * (T::KCH - c);
#pragma unroll
            for (int ks = 1; ks < 4 * T::GCH; ++ks) {
              const uint64_t aoff = (uint64_t)((ks >> 2) * (T::SLOT >> 4) + (ks & 3) * 2);
              const uint64_t boff = (uint64_t)((ks >> 2) * (T::KT * 128 >> 4) + (ks & 3) * 2);
              if (ks < nks) mma_ss(d, ad0 + aoff, bd0 + boff, idS, 1u);
            }
            commit(empty_bar(grp));
          }
          __syncwarp();
          if (++grp == T::RING_G) { grp = 0; ph ^= 1u; }
        }
        if (!ok) break;
        if (elect_one()) {
          commit(s_full + 8 * sb);
          if (i == it.ntiles - 1) commit(q_free + 8 * qb);  // this item's Q is free
        }
        __syncwarp();
        if (i > 0) pv(j - 1, prev_first, prev_k);
        prev_first = (i == 0);
        prev_k = kq;
      }
      ++kq;
    }
    if (ok && j > 0) pv(j - 1, prev_first, prev_k);
  } else if (warp >= 2) {
    // ---------------------------------------------------- softmax + epilogue
    // SPLIT threads per q row: warps w with the same w % 4 share a TMEM lane
    // quarter; quarter-mate qd owns keys [KS qd, KS qd + KS) of each tile and
    // output columns [HC qd, HC qd + HC).
    constexpr int SPLIT = T::SPLIT;
    constexpr int KS = T::KT / SPLIT;        // keys per thread per tile
    constexpr int HC = DVH / SPLIT;          // output columns per thread
    const int wq = warp & 3;
    const int qd = (warp - 2) >> 2;          // which slice of the row
    const int row = wq * 32 + lane;          // q row within the tile = TMEM lane
    const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
    // The SPLIT threads of a row meet on named barrier 1 + wq.  Such a
    // barrier waits without bound, so all of them must always reach the
    // same ones: a failed wait only clears `ok` (skipping the work that
    // depends on it), and the group leaves its loops together right after
    // the next barrier that ANDs `ok` over the group (group_and).
    auto group_and = [&](bool v) { return named_bar_and(1 + wq, 32 * SPLIT, v); };
    volatile int own_abort = 0;
    auto wait = [&](uint32_t bar, uint32_t parity, uint32_t id) {
      return waitw(bar, parity, &own_abort, id);
    };
    // The thread's TMEM stores or reads have completed (tcgen05 wait +
    // fence) before it arrives.
    auto arrive_lead = [&](uint32_t bar) { mbar_arrive(bar); };
    bool ok = true;
    int j = 0;
    for (int L = item0; L < p.n_items; L += istride) {
      const PrefillItem it = prefill_item(p, L);
      const int qi = it.q0 + row;
      int lim = p.causal ? qi + it.skv - p.Sq + 1 : it.skv;  // keys [0, lim) visible
      lim = max(0, min(it.skv, lim));
      float m_used = -INFINITY;  // log2-domain running max (lazily raised), same in the group
      float l = 0.f;             // this thread's share of the row sum

      for (int i = 0; i < it.ntiles; ++i, ++j) {
        const int sb = j & 1;
        if (ok) ok = wait(s_full + 8 * sb, (j >> 1) & 1, 30);
        float s[KS];
        float mx = -INFINITY;
        if (ok) {
          tc_fence_after();
          tmem_ld<KS>(tmem + lane_base + T::TMEM_S + sb * 128 + qd * KS, s);
          tmem_wait_ld();

          // Keys at or past `lim` are invisible to this row; only tiles that
          // straddle `lim` need the mask.  A partial last tile holds the KT
          // keys ending at skv; its keys below the tile start t0k belong to
          // the previous tile and are masked too.  The maximum is taken on
          // the raw scores (scale > 0) in 8 independent chains, then scaled
          // once.
          const int t0k = i * T::KT;
          const int kb = min(t0k, it.skv - T::KT) + qd * KS;
          if (kb + KS > lim || kb < t0k) {
#pragma unroll
            for (int c = 0; c < KS; ++c)
              if (kb + c >= lim || kb + c < t0k) s[c] = -INFINITY;
          }
          float mc[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) mc[e] = s[e];
#pragma unroll
          for (int c = 8; c < KS; ++c) mc[c & 7] = fmaxf(mc[c & 7], s[c]);
          mx = fmaxf(fmaxf(fmaxf(mc[0], mc[1]), fmaxf(mc[2], mc[3])),
                     fmaxf(fmaxf(mc[4], mc[5]), fmaxf(mc[6], mc[7])));
        }
        // row maximum over the group's slices, exchanged through shared
        // memory; the buffer alternates with the tile, so the one barrier
        // per tile also orders the reuse
        float* xb = xch + (j % T::XR) * (SPLIT * 128);
        xb[qd * 128 + row] = mx;
        ok = group_and(ok);
        if (!ok) break;
#pragma unroll
        for (int k = 0; k < SPLIT; ++k) mx = fmaxf(mx, xb[k * 128 + row]);
        mx *= p.scale_log2;
        // Raise the running max only when the tile's exceeds it by more than 8
        // (log2 units); weights stay <= 256 and O/l is unaffected.
        const bool need = mx > m_used + 8.f;
        const float m_new = need ? mx : m_used;
        const float alpha = need ? ex2(m_used - m_new) : 1.f;
        const bool warp_need = __any_sync(0xffffffffu, need);
        // a failed wait ends the tile here and the group leaves at the next group_and
        if (warp_need && i > 0) {  // rescale this thread's O columns once PV(j-1) landed
          const int t = j - 1;
          ok = wait(o_done + 8 * (t & 1), (t >> 1) & 1, 32);
          if (!ok) continue;
          tc_fence_after();
#pragma unroll 1
          for (int g = 0; g < HC / 16; ++g) {
            float o[16];
            const uint32_t ta = tmem + lane_base + T::TMEM_O + qd * HC + g * 16;
            tmem_ld16(ta, o);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 16; ++c) o[c] *= alpha;
            tmem_st16(ta, o);
          }
          tmem_wait_st();
        }
        l *= alpha;
        m_used = m_new;

        // P slice -> TMEM columns [KS/2 qd, KS/2 qd + KS/2) of S buffer sb (two
        // bf16 per column, keys in order; the whole group has read its S
        // values before the barrier above):
        // p = exp2(s * scale * log2e - m), one FMA and one SFU op per key; a row
        // that has seen no visible key yet (m = -inf) writes zeros.
        const float neg_m = m_used == -INFINITY ? 0.f : -m_used;
        const bool none = m_used == -INFINITY;
        float lc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) lc[e] = 0.f;
#pragma unroll
        for (int h16 = 0; h16 < KS / 32; ++h16) {
          float u[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int c = h16 * 32 + 2 * e;
            const float p0 = none ? 0.f : ex2(fmaf(s[c], p.scale_log2, neg_m));
            const float p1 = none ? 0.f : ex2(fmaf(s[c + 1], p.scale_log2, neg_m));
            u[e] = __uint_as_float(pack2(p0, p1, BF16));
            lc[(2 * e) & 7] += p0;
            lc[(2 * e + 1) & 7] += p1;
          }
          tmem_st16(tmem + lane_base + T::TMEM_S + sb * 128 + qd * (KS / 2) + h16 * 16, u);
        }
        l += ((lc[0] + lc[1]) + (lc[2] + lc[3])) + ((lc[4] + lc[5]) + (lc[6] + lc[7]));
        tmem_wait_st();
        tc_fence_before();
        arrive_lead(p_full + 8 * sb);
      }

      // ------------------------------------------------------ epilogue
      // row sum over the group (this round's exchange buffer is free: its
      // last readers passed the barrier of the last tile)
      float* xb = xch + (j % T::XR) * (SPLIT * 128);
      xb[qd * 128 + row] = l;
      ok = group_and(ok);
      if (!ok) break;
      float ltot = 0.f;
#pragma unroll
      for (int k = 0; k < SPLIT; ++k) ltot += xb[k * 128 + row];
      if (it.ntiles > 0) {
        const int t = j - 1;
        ok = wait(o_done + 8 * (t & 1), (t >> 1) & 1, 33);
        if (!ok) continue;  // no group barrier before the next item's first group_and
        tc_fence_after();
      }
      const float inv = ltot > 0.f ? 1.f / ltot : 0.f;
      uint8_t* orow = reinterpret_cast<uint8_t*>(p.out) +
                      ((int64_t)it.b * p.o_sb + (int64_t)it.h * p.o_sh + (int64_t)qi * p.o_ss +
                       it.part * DVH + qd * HC) * 2;
#pragma unroll 1
      for (int g = 0; g < HC / 16; ++g) {
        float o[16];
        if (it.ntiles > 0) {
          tmem_ld16(tmem + lane_base + T::TMEM_O + qd * HC + g * 16, o);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int c = 0; c < 16; ++c) o[c] = 0.f;
        }
        if (qi < p.Sq) {
          uint32_t u[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) u[e] = pack2(o[2 * e] * inv, o[2 * e + 1] * inv, BF16);
          uint4* dst = reinterpret_cast<uint4*>(orow + g * 32);
          dst[0] = make_uint4(u[0], u[1], u[2], u[3]);
          dst[1] = make_uint4(u[4], u[5], u[6], u[7]);
        }
      }
      if (it.ntiles > 0) {  // O may now be overwritten by the next item's PV
        tc_fence_before();
        arrive_lead(o_free);
      }
      if (qd == 0 && it.part == 0 && p.lse && qi < p.Sq)
        p.lse[((int64_t)it.b * p.Hq + it.h) * p.Sq + qi] =
            ltot > 0.f ? (m_used + __log2f(ltot)) * 0.69314718055994531f : -INFINITY;
    }
    if (!ok) *abort_flag = 1;
  }
  abort_tail(abort_flag, warp, drain);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, T::TMEM_COLS);
  }
}

}  // namespace attn
