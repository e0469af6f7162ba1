// prefill_ab_kernel.cuh -- causal (or full) prefill at d_k = d_v = 512 on SM
// pairs that split the two matmuls between them.
//
// At head_dim 512 a 128-row fp32 O tile fills all 512 TMEM columns of an
// SM, leaving none for S.  Instead of splitting d_v into halves that each
// recompute S = Q K^T (1.5x the MMA work), a cluster of two CTAs on two SMs
// takes one work item (128 query rows of one head, all 512 output columns)
// and gives each SM one matmul:
//
//   CTA 0 ("scores"):  Q (bf16/fp16) in TMEM columns 256..511, copied there
//       once per item; S[128 x 128 keys] = Q K^T by TMEM-operand UMMAs into
//       two S buffers (columns 0..255); the online softmax (one thread per
//       query row and 64-key half of the tile) turns each half of S into P,
//       writes it into that half's local staging buffer and ships it to
//       CTA 1's shared memory with bulk copies (one 4 KB copy per warp: its
//       32 rows).
//   CTA 1 ("output"):  O[128 x 512] in all of its TMEM; O += P V over each
//       64-key half (two UMMAs of N = 256); when a row's running maximum
//       was raised it rescales O in TMEM first; at the end of the item
//       O / l -> out.
//
// Every FLOP of the two matmuls is done once, and each SM streams one
// operand: CTA 0 the K tiles (128 keys x 4 chunks per copy), CTA 1 the V
// halves (64 keys x 8 chunks per copy): 64 KB boxes, since one SM's TMA
// copies run at about two boxes per microsecond whatever their size.
// ("GQA和MLA详解" section 1: prefill is the quadratic, compute-bound phase;
// "带你了解Attention" section 6.3: tiling with an online softmax.)
//
// Roles (608 threads per CTA):
//   CTA 0: warp 0 lane 0 copies Q and K (TMA); warp 1 copies Q into TMEM
//       and issues the S UMMAs; warps 2-9 run the softmax (warp w: TMEM lane
//       quarter w % 4, tile half (w - 2) / 4); warps 10-18 are idle.
//   CTA 1: warp 0 lane 0 copies V; warp 1 issues the PV UMMAs and posts
//       events (rescale, end of item) to warps 2-17, which rescale O or
//       write the output; warp 18 watches the P buffers fill and tells CTA
//       0 when a staged half has landed.
// Cross-CTA traffic: P by cp.async.bulk from CTA 0's staging buffers (on
// this part a bulk copy moves shared memory to the peer SM about twice as
// fast as st.async), rescale factors, the halves' row sums and the row
// maxima by st.async (all bytes counted on CTA 1 mbarriers); "P buffer
// free" by tcgen05.commit multicast from CTA 1's MMA issuer; "staging
// buffer landed" and "row sums read" by relaxed remote arrivals from CTA 1.
// All waits are bounded; the two CTAs meet in a hardware cluster barrier
// only after both have left every loop.
#pragma once

#include "prefill_kernel.cuh"

namespace attn {

struct PrefillABTraits {
  static constexpr int DK = 512, DV = 512;
  static constexpr int TILE = 128;               // q rows per item (MMA M)
  static constexpr int KT = 128;                 // keys per S tile (MMA N of S)
  static constexpr int HT = 64;                  // keys per PV step (half an S tile)
  static constexpr int SLOT = 65536;             // one copy: 4 chunks x 128 rows or 8 x 64
  static constexpr int CHUNK_Q = 16384;          // [128 rows x 64 columns] of Q or K
  static constexpr int CHUNK_V = 8192;           // [64 keys x 64 columns] of V
  static constexpr int RING = 3;                 // CTA 0: Q/K copies in flight
  static constexpr int RING_V = 2;               // CTA 1: V copies in flight
  static constexpr int NPB = 4;                  // CTA 1: P half buffers (two tiles)
  static constexpr int SM_WARPS = 8;             // CTA 0: softmax warps 2..9, a q row per thread and half
  static constexpr int SPLIT = 4;                // CTA 1: output threads per q row
  static constexpr int WORK_WARPS = 4 * SPLIT;   // CTA 1: output warps 2..17
  static constexpr int RELAY_WARP = 2 + WORK_WARPS;         // CTA 1: P arrivals -> CTA 0
  static constexpr int THREADS = 64 + 32 * WORK_WARPS + 32;
  static constexpr int PH_BYTES = TILE * HT * 2;           // one P half: 16 KB
  // bytes landing in P buffer b: a tile's first half (even b) comes with the
  // rows' rescale factors, its second half (odd b) needs none
  static constexpr int PMSG_BYTES = PH_BYTES + TILE * 4;
  __host__ __device__ static constexpr int pmsg_bytes(int b) { return (b & 1) ? PH_BYTES : PMSG_BYTES; }
  static constexpr int PQ_BYTES = PH_BYTES / 4;            // one 32-row quarter of a P half
  static constexpr int L_BYTES = 3 * TILE * 4;             // the halves' row sums + row maxima
  // CTA 0: ring of RING slots, two P half staging buffers.  CTA 1: ring of
  // RING_V slots, the P half buffers (K-major, 128-byte swizzle) where CTA
  // 0's third slot lies, rescale factors, row sums and maxima.
  static constexpr int OFF_RING = 0;
  static constexpr int OFF_P = OFF_RING + RING_V * SLOT;
  static constexpr int OFF_SIDE = OFF_RING + RING * SLOT;
  static constexpr int OFF_STAGE = OFF_SIDE;               // CTA 0: [2][PH_BYTES]
  static constexpr int OFF_ALPHA = OFF_SIDE;               // CTA 1: float [NPB][128]
  static constexpr int OFF_L = OFF_ALPHA + NPB * TILE * 4; // CTA 1: float [2][128] row sums by half
  static constexpr int OFF_M = OFF_L + 2 * TILE * 4;       // CTA 1: float [128] row maxima (log2)
  static constexpr int OFF_EV = OFF_SIDE + 2 * PH_BYTES;  // CTA 1: event {type, arg0, arg1, arg2}
  static constexpr int OFF_FLAGS = OFF_EV + 16;            // int [4]: abort, tmem
  static constexpr int OFF_BAR = OFF_FLAGS + 16;
  // full[3] empty[3] s_full[2] s_free[2] q_cp p_free[4] p_full[4] o_item
  // o_sync ev_go ev_done l_full drain stage_free[2] l_free (the same layout
  // in both CTAs: p_free is reached by a multicast commit, the others by
  // mapa)
  static constexpr int NBAR = 2 * RING + 2 + 2 + 1 + 2 * NPB + 1 + 1 + 1 + 1 + 1 + 1 + 2 + 1;
  static constexpr int SMEM_BYTES = OFF_BAR + NBAR * 8 + 1024;
  static constexpr int TMEM_S = 0;               // CTA 0: S buffers, 128 columns each
  static constexpr int TMEM_Q = 256;             // CTA 0: Q, 8 columns per 16-element K step
  static constexpr int TMEM_O = 0;               // CTA 1: O, 512 columns
  static_assert(OFF_P + NPB * PH_BYTES == OFF_SIDE, "CTA 1's P buffers end where CTA 0's ring does");
  static_assert(OFF_M + TILE * 4 <= OFF_EV && OFF_STAGE % 1024 == 0, "side buffers");
  static_assert(NPB % 2 == 0, "a tile's two halves take consecutive P buffers");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

// CTA 1's event queue (one slot): posted by its MMA issuer, handled by its
// warps 2.., which arrive on ev_done before the next event is posted.
enum : int { AB_EV_RESCALE = 1, AB_EV_OUTPUT = 2, AB_EV_EMPTY = 3, AB_EV_STOP = 4 };

template <bool BF16>
__global__ void __launch_bounds__(PrefillABTraits::THREADS, 1)
    prefill_ab_kernel(const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
  using T = PrefillABTraits;
  const uint32_t cr = cluster_ctarank();  // 0: scores, 1: output
  const int item0 = (int)(blockIdx.x >> 1);
  const int istride = (int)(gridDim.x >> 1);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t ring = sbase + T::OFF_RING;
  const uint32_t pbuf = sbase + T::OFF_P;
  const uint32_t stage = sbase + T::OFF_STAGE;                      // CTA 0
  float* alpha_sm = reinterpret_cast<float*>(smem + T::OFF_ALPHA);  // CTA 1
  float* l_sm = reinterpret_cast<float*>(smem + T::OFF_L);          // CTA 1
  float* m_sm = reinterpret_cast<float*>(smem + T::OFF_M);          // CTA 1
  volatile int* ev = reinterpret_cast<volatile int*>(smem + T::OFF_EV);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + T::OFF_FLAGS);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + T::OFF_FLAGS + 4);
  const uint32_t bar0 = sbase + T::OFF_BAR;
  auto full_bar = [&](int g) { return bar0 + 8u * g; };
  auto empty_bar = [&](int g) { return bar0 + 8u * (T::RING + g); };
  const uint32_t s_full = bar0 + 8u * (2 * T::RING);  // [2] CTA 0
  const uint32_t s_free = s_full + 16;                // [2] CTA 0
  const uint32_t q_cp = s_free + 16;                  // CTA 0: Q in TMEM
  const uint32_t p_free = q_cp + 8;                   // [NPB] CTA 0: P half buffer free in CTA 1
  const uint32_t p_full = p_free + 8 * T::NPB;        // [NPB] CTA 1: P half + factors landed
  const uint32_t o_item = p_full + 8 * T::NPB;        // CTA 1: an item's last PV completed
  const uint32_t o_sync = o_item + 8;                 // CTA 1: every PV issued so far completed
  const uint32_t ev_go = o_sync + 8;                  // CTA 1: event posted
  const uint32_t ev_done = ev_go + 8;                 // CTA 1: event handled
  const uint32_t l_full = ev_done + 8;                // CTA 1: row sums and maxima landed
  const uint32_t drain = l_full + 8;
  const uint32_t stage_free = drain + 8;              // [2] CTA 0: a staged P half has landed in CTA 1
  const uint32_t l_free = stage_free + 16;            // CTA 0: CTA 1 has read the row sums

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int g = 0; g < T::RING; ++g) {
      mbar_init(full_bar(g), 1);
      mbar_init(empty_bar(g), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full + 8 * i, 1);
      mbar_init(s_free + 8 * i, T::SM_WARPS);
    }
    for (int i = 0; i < T::NPB; ++i) {
      mbar_init(p_free + 8 * i, 1);
      mbar_init(p_full + 8 * i, 1);
    }
    mbar_init(q_cp, 1);
    mbar_init(o_item, 1);
    mbar_init(o_sync, 1);
    mbar_init(ev_go, 1);
    mbar_init(ev_done, T::WORK_WARPS);
    mbar_init(l_full, 1);
    mbar_init(drain, 1);
    mbar_init(stage_free, 1);
    mbar_init(stage_free + 8, 1);
    mbar_init(l_free, 1);
    *abort_flag = 0;
    fence_mbar_init();
    if (cr == 1) {  // the first NPB P halves and the first item's row sums
      for (int i = 0; i < T::NPB; ++i) mbar_arrive_expect_tx(p_full + 8 * i, T::pmsg_bytes(i));
      mbar_arrive_expect_tx(l_full, T::L_BYTES);
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers exist
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint64_t tmo = p.timeout_ns;

  if (cr == 0 && warp == 0 && lane == 0) {
    // ---------------------------------------------------- CTA 0: Q and K copies
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    const uint64_t pol_q = l2_policy_evict_first();
    const uint64_t pol_k = l2_policy_evict_last();  // K tiles serve every head of the group
    int grp = 0;
    uint32_t ph = 0;
    bool ok = true;
    auto load = [&](const CUtensorMap* map, int row, int ch, int h, int b, uint64_t pol) {
      if (!ok) return;
      ok = mbar_wait(empty_bar(grp), ph ^ 1u, abort_flag, tmo, 70);
      if (!ok) return;
      mbar_arrive_expect_tx(full_bar(grp), T::SLOT);
      tma_load_5d(ring + grp * T::SLOT, map, full_bar(grp), 0, row, ch, h, b, pol);
      if (++grp == T::RING) { grp = 0; ph ^= 1u; }
    };
    for (int L = item0; L < p.n_items && ok; L += istride) {
      const PrefillItem it = prefill_item(p, L);
      if (it.ntiles == 0) continue;
      load(&tmQ, it.q0, 0, it.h, it.b, pol_q);
      load(&tmQ, it.q0, 4, it.h, it.b, pol_q);
      for (int t = 0; t < it.ntiles && ok; ++t) {
        // a partial last tile is read as the 128 keys ending at skv (the
        // rows before the tile start are masked), so no row past skv is read
        const int win0 = min(t * T::KT, it.skv - T::KT);
        load(&tmK, win0, 0, it.kvh, it.b, pol_k);
        load(&tmK, win0, 4, it.kvh, it.b, pol_k);
      }
    }
  } else if (cr == 1 && warp == 0 && lane == 0) {
    // ---------------------------------------------------- CTA 1: V copies
    tma_prefetch_desc(&tmV);
    const uint64_t pol_v = l2_policy_evict_last();
    int grp = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int L = item0; L < p.n_items && ok; L += istride) {
      const PrefillItem it = prefill_item(p, L);
      for (int t = 0; t < it.ntiles && ok; ++t) {
        const int win0 = min(t * T::KT, it.skv - T::KT);
        for (int hh = 0; hh < 2 && ok; ++hh) {
          ok = mbar_wait(empty_bar(grp), ph ^ 1u, abort_flag, tmo, 71);
          if (!ok) break;
          mbar_arrive_expect_tx(full_bar(grp), T::SLOT);
          tma_load_5d(ring + grp * T::SLOT, &tmV, full_bar(grp), 0, win0 + hh * T::HT, 0, it.kvh,
                      it.b, pol_v);
          if (++grp == T::RING_V) { grp = 0; ph ^= 1u; }
        }
      }
    }
  } else if (cr == 0 && warp == 1) {
    // ---------------------------------------------------- CTA 0: Q -> TMEM, S UMMAs
    constexpr uint32_t idS = umma_idesc(128, T::KT, BF16, false, false);  // Q, K both K-major
    int grp = 0;
    uint32_t ph = 0;
    bool ok = true;
    int j = 0, kq = 0;
    for (int L = item0; L < p.n_items && ok; L += istride) {
      const PrefillItem it = prefill_item(p, L);
      if (it.ntiles == 0) continue;
      // the previous item's S UMMAs read TMEM Q: wait for the last of them
      if (j > 0) ok = mbar_wait_warp(s_full + 8 * ((j - 1) & 1), ((j - 1) >> 1) & 1, abort_flag, tmo, 72);
      // Q chunks c = 0..7 -> TMEM columns TMEM_Q + 8 (4 c + ks), one
      // 128-row x 32-byte copy per 16-element K step
      for (int qs = 0; qs < 2 && ok; ++qs) {
        ok = mbar_wait_warp(full_bar(grp), ph, abort_flag, tmo, 73);
        if (!ok) break;
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint64_t sd = umma_sdesc(ring + grp * T::SLOT + c * T::CHUNK_Q, 16, 1024, SMEM_SW128);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              tmem_cp_128x256b(tmem + T::TMEM_Q + 8 * (4 * (4 * qs + c) + ks), sd + 2 * ks);
          }
          umma_commit(empty_bar(grp));
        }
        __syncwarp();
        if (++grp == T::RING) { grp = 0; ph ^= 1u; }
      }
      if (!ok) break;
      if (elect_one()) umma_commit(q_cp);
      __syncwarp();
      ok = mbar_wait_warp(q_cp, kq & 1, abort_flag, tmo, 74);
      if (!ok) break;
      tc_fence_after();
      ++kq;
      for (int t = 0; t < it.ntiles && ok; ++t, ++j) {
        const int sb = j & 1;
        if (j >= 2) ok = mbar_wait_warp(s_free + 8 * sb, ((j >> 1) - 1) & 1, abort_flag, tmo, 75);
        if (!ok) break;
        tc_fence_after();
        for (int kh = 0; kh < 2 && ok; ++kh) {  // K chunks 4 kh .. 4 kh + 3
          ok = mbar_wait_warp(full_bar(grp), ph, abort_flag, tmo, 76);
          if (!ok) break;
          tc_fence_after();
          if (elect_one()) {
            const uint32_t d = tmem + T::TMEM_S + sb * 128;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              // B = K chunk: K-major, 128-byte swizzle, 8-key groups 1024
              // bytes apart, 32 bytes per K step; A = Q from TMEM
              const uint64_t bd = umma_sdesc(ring + grp * T::SLOT + c * T::CHUNK_Q, 16, 1024, SMEM_SW128);
#pragma unroll
              for (int ks = 0; ks < 4; ++ks)
                umma_ts(d, tmem + T::TMEM_Q + 8 * (4 * (4 * kh + c) + ks), bd + 2 * ks, idS,
                        (kh | c | ks) ? 1u : 0u);
            }
            umma_commit(empty_bar(grp));
          }
          __syncwarp();
          if (++grp == T::RING) { grp = 0; ph ^= 1u; }
        }
        if (!ok) break;
        if (elect_one()) umma_commit(s_full + 8 * sb);
        __syncwarp();
      }
    }
    if (!ok) *abort_flag = 1;
  } else if (cr == 1 && warp == 1) {
    // ---------------------------------------------------- CTA 1: PV UMMAs, events
    constexpr uint32_t idO = umma_idesc(128, 256, BF16, false, true);  // P K-major, V MN-major
    int grp = 0;
    uint32_t ph = 0;
    bool ok = true;
    int h = 0, ne = 0, nsync = 0;  // half tiles, events posted, o_sync phases
    const uint32_t l_free_0 = mapa_shared(l_free, 0);
    bool out_pending = false;  // an item's output event not yet seen handled
    // wait until the last event posted was handled; once an item's output
    // has been written, its row sums are read: CTA 0 may send the next ones
    auto wait_done = [&](uint32_t id) {
      ok = mbar_wait_warp(ev_done, (ne - 1) & 1, abort_flag, tmo, id);
      if (ok && out_pending) {
        if (lane == 0) mbar_arrive_remote_relaxed(l_free_0);
        __syncwarp();
        out_pending = false;
      }
    };
    // one event at a time: wait until the previous one was handled
    auto post = [&](int type, int a0, int a1, int a2) {
      if (!ok) return;
      if (ne > 0) wait_done(77);
      if (!ok) return;
      if (lane == 0) {
        ev[0] = type;
        ev[1] = a0;
        ev[2] = a1;
        ev[3] = a2;
        mbar_arrive(ev_go);
      }
      __syncwarp();
      ++ne;
    };
    for (int L = item0; L < p.n_items && ok; L += istride) {
      const PrefillItem it = prefill_item(p, L);
      if (it.ntiles == 0) {
        post(AB_EV_EMPTY, L, 0, 0);
        continue;
      }
      for (int t = 0; t < it.ntiles && ok; ++t) {
        for (int hh = 0; hh < 2 && ok; ++hh, ++h) {
          const int pb = h % T::NPB;
          const bool first = t == 0 && hh == 0;
          ok = mbar_wait_warp_cluster(p_full + 8 * pb, (h / T::NPB) & 1, abort_flag, tmo, 78);
          if (!ok) break;
          // rows whose running maximum was raised at this tile: O *= alpha
          // before its first half (the factors come with that half; the
          // first half of an item overwrites O, so needs none)
          bool rescale = false;
          if (!first && hh == 0) {
            const float4 a4 = *reinterpret_cast<const float4*>(alpha_sm + pb * T::TILE + 4 * lane);
            rescale = __any_sync(0xffffffffu, a4.x != 1.f || a4.y != 1.f || a4.z != 1.f || a4.w != 1.f);
          }
          if (rescale) {
            // every PV so far has landed (a commit tracks all earlier UMMAs)
            if (elect_one()) umma_commit(o_sync);
            __syncwarp();
            ok = mbar_wait_warp(o_sync, nsync & 1, abort_flag, tmo, 79);
            ++nsync;
            post(AB_EV_RESCALE, pb, 0, 0);
            if (ok) wait_done(80);
            if (!ok) break;
            tc_fence_after();
          }
          if (first && ne > 0) {  // the previous event (an item's output) read O out of TMEM
            wait_done(81);
            if (!ok) break;
            tc_fence_after();
          }
          ok = mbar_wait_warp(full_bar(grp), ph, abort_flag, tmo, 82);
          if (!ok) break;
          tc_fence_after();
          fence_proxy_async_smem();  // the st.async P rows, for the MMA's operand reads
          if (elect_one()) {
            // the next use of this P buffer (half h + NPB)
            mbar_arrive_expect_tx(p_full + 8 * pb, T::pmsg_bytes(pb));
            // A = P half: K-major, 128-byte swizzle, 32 bytes per K step.
            // B = V half [8 chunks][64 keys][64 columns]: MN-major, 128-byte
            // swizzle, 64-column chunks 8 KB apart (LBO), 8-key groups 1024
            // bytes apart (SBO), 16 keys per K step = 2048 bytes.
            const uint64_t ad = umma_sdesc(pbuf + pb * T::PH_BYTES, 16, 1024, SMEM_SW128);
#pragma unroll
            for (int dn = 0; dn < 2; ++dn) {
              const uint64_t bd =
                  umma_sdesc(ring + grp * T::SLOT + dn * 4 * T::CHUNK_V, T::CHUNK_V, 1024, SMEM_SW128);
#pragma unroll
              for (int ks = 0; ks < 4; ++ks)
                umma_ss(tmem + T::TMEM_O + dn * 256, ad + 2 * ks, bd + (uint64_t)(ks * (2048 >> 4)),
                        idO, (first && ks == 0) ? 0u : 1u);
            }
            umma_commit(empty_bar(grp));
            umma_commit_mc(p_free + 8 * pb, 3);  // both CTAs: this P buffer is free
            if (t == it.ntiles - 1 && hh == 1) umma_commit(o_item);  // the item's O is complete
          }
          __syncwarp();
          if (++grp == T::RING_V) { grp = 0; ph ^= 1u; }
        }
      }
      if (ok) {
        post(AB_EV_OUTPUT, L, h - 1, 0);
        out_pending = true;
      }
    }
    post(AB_EV_STOP, 0, 0, 0);
    if (!ok) *abort_flag = 1;
  } else if (cr == 0 && warp >= 2 && warp < 2 + T::SM_WARPS) {
    // ---------------------------------------------------- CTA 0: softmax
    // Warp w reads TMEM lane quarter w % 4 (32 q rows) and owns 64-key half
    // hh = (w - 2) / 4 of every tile.  Each thread takes its row's maximum
    // over the whole tile itself (the two warps of a quarter do it twice
    // rather than exchange it), then the weights of its half, written into
    // the half's staging buffer and shipped by one 4 KB bulk copy per warp
    // (its 32 rows are contiguous in the P layout).
    const int wq = warp & 3;
    const int hh = (warp - 2) >> 2;
    const int row = wq * 32 + lane;
    const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
    volatile int own_abort = 0;
    const uint32_t p_full_1 = mapa_shared(p_full, 1);
    const uint32_t pbuf_1 = mapa_shared(pbuf, 1);
    const uint32_t alpha_1 = mapa_shared(smem_u32(alpha_sm), 1);
    const uint32_t l_1 = mapa_shared(smem_u32(l_sm), 1);
    const uint32_t m_1 = mapa_shared(smem_u32(m_sm), 1);
    const uint32_t l_full_1 = mapa_shared(l_full, 1);
    // P half layout, the same in a staging buffer and in CTA 1's P buffers:
    // K-major, 128-byte swizzle, 16-byte unit v of row r at 128 r + ((v ^
    // (r & 7)) * 16)
    const uint32_t sbuf = stage + hh * T::PH_BYTES + row * 128;
    bool ok = true;
    int j = 0, nitem = 0;
    for (int L = item0; L < p.n_items && ok; L += istride) {
      const PrefillItem it = prefill_item(p, L);
      if (it.ntiles == 0) continue;  // CTA 1 writes the empty item
      const int qi = it.q0 + row;
      int lim = p.causal ? qi + it.skv - p.Sq + 1 : it.skv;  // keys [0, lim) visible
      lim = max(0, min(it.skv, lim));
      float m_used = -INFINITY;  // log2-domain running max
      float la[4] = {0.f, 0.f, 0.f, 0.f};  // the half's row sum, in four independent parts
      for (int t = 0; t < it.ntiles && ok; ++t, ++j) {
        const int sb = j & 1;
        const int h = 2 * j + hh;   // P half index
        const int pb = h % T::NPB;  // CTA 1's P buffer
        const uint32_t srow = tmem + lane_base + T::TMEM_S + sb * 128;
        ok = mbar_wait_warp(s_full + 8 * sb, (j >> 1) & 1, &own_abort, tmo, 83);
        if (!ok) break;
        tc_fence_after();
        const int tile0 = t * T::KT;
        const int win0 = min(tile0, it.skv - T::KT);
        // a tile wholly inside [0, lim) for this row: no mask, and a quarter
        // of its exponentials go to the FMA pipe.  Column c of the tile is
        // key win0 + c (a shifted last window's keys below tile0 belong to
        // the previous tile).
        const bool whole = win0 == tile0 && tile0 + T::KT <= lim;
        // pass 1: the row maximum of the raw scores over the tile (scale > 0
        // keeps the order), in two 64-column loads (each wait for TMEM data
        // costs about as much as folding 64 values)
        float mx = -INFINITY;
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          float v[64];
          tmem_ld<64>(srow + 64 * c, v);
          tmem_wait_ld();
          if (whole) {
#pragma unroll
            for (int e = 0; e < 64; e += 2) mx = fmaxf(mx, fmaxf(v[e], v[e + 1]));
          } else {
#pragma unroll
            for (int e = 0; e < 64; ++e) {
              const int key = win0 + 64 * c + e;
              if (key >= tile0 && key < lim) mx = fmaxf(mx, v[e]);
            }
          }
        }
        const float tm = mx * p.scale_log2;
        // lazy raise (threshold 8 in log2 units): the weights stay <= 256
        const bool need = tm > m_used + 8.f;
        const float mn = need ? tm : m_used;
        const float alpha = need ? ex2(m_used - mn) : 1.f;  // m_used = -inf: 0
        m_used = mn;
#pragma unroll
        for (int k = 0; k < 4; ++k) la[k] *= alpha;
        // an invisible key's weight is exactly 0; a row with no visible key
        // yet keeps m_used = -inf and all weights 0
        const float neg_mu = m_used == -INFINITY ? 0.f : -m_used;
        // pass 2: this half's weights.  The staging buffer last held the
        // previous tile's half: CTA 1 reports when it landed.
        if (j >= 1) ok = mbar_wait_warp(stage_free + 8 * hh, (j - 1) & 1, &own_abort, tmo, 91);
        if (!ok) break;
        {
          float v[2][32];
          tmem_ld<32>(srow + hh * T::HT, v[0]);
          tmem_ld<32>(srow + hh * T::HT + 32, v[1]);
          tmem_wait_ld();
          // S buffer sb has been read by this warp
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(s_free + 8 * sb);
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t u[16];
            if (whole) {
#pragma unroll
              for (int e = 0; e < 32; e += 2) {
                const float p0 = ex2(fmaf(v[c][e], p.scale_log2, neg_mu));
                const float x1 = fmaf(v[c][e + 1], p.scale_log2, neg_mu);
                const float p1 = (e & 2) ? ex2_fma(x1) : ex2(x1);
                la[(e >> 1) & 3] += p0 + p1;
                u[e / 2] = pack2(p0, p1, BF16);
              }
            } else {
#pragma unroll
              for (int e = 0; e < 32; e += 2) {
                const int key = win0 + hh * T::HT + 32 * c + e;
                const float p0 = (key >= tile0 && key < lim) ? ex2(fmaf(v[c][e], p.scale_log2, neg_mu)) : 0.f;
                const float p1 =
                    (key + 1 >= tile0 && key + 1 < lim) ? ex2(fmaf(v[c][e + 1], p.scale_log2, neg_mu)) : 0.f;
                la[(e >> 1) & 3] += p0 + p1;
                u[e / 2] = pack2(p0, p1, BF16);
              }
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int unit = 4 * c + k;  // 8 keys per 16-byte unit
              st_shared_v4(sbuf + ((unit ^ (row & 7)) << 4), u[4 * k], u[4 * k + 1], u[4 * k + 2],
                           u[4 * k + 3]);
            }
          }
        }
        fence_proxy_async_smem();  // for the bulk copy's reads
        // CTA 1's P buffer pb and its rescale factors were last read by PV(h - NPB)
        if (h >= T::NPB)
          ok = mbar_wait_warp_cluster(p_free + 8 * pb, ((h / T::NPB) - 1) & 1, &own_abort, tmo, 84);
        __syncwarp();  // every lane's row is staged
        if (!ok) break;
        const uint32_t bar = p_full_1 + 8 * pb;
        if (lane == 0)
          bulk_copy_to_peer(pbuf_1 + pb * T::PH_BYTES + wq * T::PQ_BYTES,
                            stage + hh * T::PH_BYTES + wq * T::PQ_BYTES, T::PQ_BYTES, bar);
        // O's rescale factor before the tile's first PV
        if (hh == 0) st_async_f32(alpha_1 + (pb * T::TILE + row) * 4, alpha, bar);
      }
      if (!ok) break;
      // the half's row sum (and the row maximum), once CTA 1 has read the
      // previous item's
      if (nitem > 0) ok = mbar_wait_warp_cluster(l_free, (nitem - 1) & 1, &own_abort, tmo, 92);
      if (!ok) break;
      ++nitem;
      st_async_f32(l_1 + (hh * T::TILE + row) * 4, (la[0] + la[1]) + (la[2] + la[3]), l_full_1);
      if (hh == 0) st_async_f32(m_1 + row * 4, m_used, l_full_1);
    }
    if (!ok) *abort_flag = 1;
  } else if (cr == 1 && warp >= 2 && warp < T::RELAY_WARP) {
    // ---------------------------------------------------- CTA 1: rescale, output
    // Four threads per row (warps with the same warp % 4 share a TMEM lane
    // quarter), each owning 128 of the row's 512 output columns.
    const int wq = warp & 3;
    const int qd = (warp - 2) >> 2;
    const int row = wq * 32 + lane;
    const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
    constexpr int HC = T::DV / T::SPLIT;  // 128 columns per thread
    volatile int own_abort = 0;
    bool ok = true;
    int e = 0, nl = 0;  // events handled, row-sum messages consumed
    for (;;) {
      ok = mbar_wait_warp(ev_go, e & 1, &own_abort, tmo, 85);
      if (!ok) break;
      const int type = ev[0], a0 = ev[1];
      ++e;
      if (type == AB_EV_STOP) {
        __syncwarp();
        if (lane == 0) mbar_arrive(ev_done);
        break;
      }
      if (type == AB_EV_RESCALE) {
        const float a = alpha_sm[a0 * T::TILE + row];
        tc_fence_after();
        // TMEM loads and stores are warp-collective: the whole warp takes
        // part if any of its rows needs the factor
        if (__any_sync(0xffffffffu, a != 1.f)) {
#pragma unroll 1
          for (int c0 = 0; c0 < HC; c0 += 16) {
            float o[16];
            const uint32_t ta = tmem + lane_base + T::TMEM_O + qd * HC + c0;
            tmem_ld16(ta, o);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 16; ++c) o[c] *= a;
            tmem_st16(ta, o);
          }
          tmem_wait_st();
        }
        tc_fence_before();
      } else {  // AB_EV_OUTPUT, AB_EV_EMPTY: O / l -> out for item a0
        const PrefillItem it = prefill_item(p, a0);
        const int qi = it.q0 + row;
        float inv = 0.f, lse = -INFINITY;
        if (type == AB_EV_OUTPUT) {
          ok = mbar_wait_warp(o_item, nl & 1, &own_abort, tmo, 86) &&
               mbar_wait_warp_cluster(l_full, nl & 1, &own_abort, tmo, 87);
          if (ok) {
            tc_fence_after();
            const float lt = l_sm[row] + l_sm[T::TILE + row];
            inv = lt > 0.f ? 1.f / lt : 0.f;
            if (lt > 0.f) lse = (m_sm[row] + __log2f(lt)) * 0.69314718055994531f;
          }
        }
        if (ok && qd == 0 && p.lse && qi < p.Sq)
          p.lse[((int64_t)it.b * p.Hq + it.h) * p.Sq + qi] = lse;
        if (ok) {  // warp-uniform: the TMEM loads are warp-collective
          uint8_t* orow = reinterpret_cast<uint8_t*>(p.out) +
                          ((int64_t)it.b * p.o_sb + (int64_t)it.h * p.o_sh + (int64_t)qi * p.o_ss +
                           qd * HC) * 2;
#pragma unroll 1
          for (int c0 = 0; c0 < HC; c0 += 32) {
            float o[32];
            if (type == AB_EV_OUTPUT) {
              tmem_ld16(tmem + lane_base + T::TMEM_O + qd * HC + c0, *reinterpret_cast<float(*)[16]>(o));
              tmem_ld16(tmem + lane_base + T::TMEM_O + qd * HC + c0 + 16,
                        *reinterpret_cast<float(*)[16]>(o + 16));
              tmem_wait_ld();
            } else {
#pragma unroll
              for (int c = 0; c < 32; ++c) o[c] = 0.f;
            }
            if (qi < p.Sq) {  // rows past Sq (a partial last q tile) are not stored
              uint32_t u[16];
#pragma unroll
              for (int c = 0; c < 16; ++c) u[c] = pack2(o[2 * c] * inv, o[2 * c + 1] * inv, BF16);
              uint4* dst = reinterpret_cast<uint4*>(orow + c0 * 2);
#pragma unroll
              for (int v = 0; v < 4; ++v) dst[v] = make_uint4(u[4 * v], u[4 * v + 1], u[4 * v + 2], u[4 * v + 3]);
            }
          }
        }
        if (type == AB_EV_OUTPUT) {
          tc_fence_before();
          // row sums consumed: arm the next item's (CTA 0 sends them only
          // after the MMA issuer has seen every warp arrive on ev_done and
          // told it so through l_free)
          if (ok && threadIdx.x == 64) mbar_arrive_expect_tx(l_full, T::L_BYTES);
          ++nl;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(ev_done);
      if (!ok) break;
    }
    if (!ok) *abort_flag = 1;
  } else if (cr == 1 && warp == T::RELAY_WARP) {
    // ---------------------------------------------------- CTA 1: P arrivals -> CTA 0
    // Watches the P buffers fill, in order, and tells CTA 0 as soon as a
    // half has landed, so that its staging buffer can take the next one.
    // (The MMA issuer waits on the same barriers; a phase cannot complete
    // twice before this warp sees it, since the copies that would complete
    // it next come from a staging buffer this warp must free first.)
    const uint32_t stage_free_0 = mapa_shared(stage_free, 0);
    bool ok = true;
    int h = 0;
    for (int L = item0; L < p.n_items && ok; L += istride) {
      const PrefillItem it = prefill_item(p, L);
      for (int hh = 0; hh < 2 * it.ntiles && ok; ++hh, ++h) {
        ok = mbar_wait_warp_cluster(p_full + 8 * (h % T::NPB), (h / T::NPB) & 1, abort_flag, tmo, 93);
        if (ok && lane == 0) mbar_arrive_remote_relaxed(stage_free_0 + 8 * (h & 1));
        __syncwarp();
      }
    }
    if (!ok) *abort_flag = 1;
  }

  // Common exit.  After a give-up, issued UMMAs, copies and st.async bytes
  // must land before the pair leaves: the MMA warps commit and wait (bounded)
  // for a drain barrier, thread 0 gives copies 2 ms; then both CTAs meet.
  __syncthreads();
  if (*abort_flag) {
    if (warp == 1) {
      if (elect_one()) umma_commit(drain);
      __syncwarp();
      volatile int never = 0;
      mbar_wait_warp(drain, 0, &never, 1000000ull, 88);
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
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace attn
