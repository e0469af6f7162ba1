// prefill_kernel.cuh -- causal (or full) attention forward for Sq > 1.
//
// Prefill is the quadratic phase ("GQA和MLA详解" section 1: T enters both
// matmuls as M and N) and is compute-bound, so both matmuls run on the
// tensor cores.  The T x T score matrix is never materialised: keys are
// streamed in tiles of 128 with an online softmax ("带你了解Attention"
// section 6.3, FlashAttention: tiling plus online softmax; "GQA和MLA详解"
// section 4, shared-memory tiling).
//
// One CTA owns 128 query rows of one head and DVH output columns:
//
//   S[128 x 128]   = Q_tile[128 x d_k] * K_tile^T            (tcgen05 -> TMEM)
//   P = exp2(S*scale*log2e - m), row max m kept per thread (thread = row)
//   O[128 x DVH]  += P[128 x 128] * V_tile[128 x DVH]        (tcgen05 -> TMEM)
//
// TMEM holds 512 fp32 columns per SM.  Two S buffers (256 columns) plus a
// 128 x 512 fp32 O would need 768, so at d_v = 512 two CTAs share a q tile,
// each owning half of d_v (DVH = 256) and each recomputing S.  The K/V
// tiles those two CTAs (and the G heads of the group) read are the same, so
// they come from L2.
//
// Warp roles (192 threads): warp 0 issues TMA loads (Q once, then K/V tiles
// through a ring of 16 KB chunk slots), warp 1 allocates TMEM and issues
// UMMA, warps 2-5 run the softmax, rescale and epilogue (thread = q row).
#pragma once

#include "sm100.cuh"

namespace attn {

struct PrefillParams {
  void* out;                  // [B, Hq, Sq, d_v]
  int64_t o_sb, o_sh, o_ss;   // element strides of out
  float* lse;                 // [B, Hq, Sq] or NULL
  const int32_t* skv;         // [B] (device)
  int B, Hq, Hkv, G, Sq;
  int n_qtiles, dv_parts;
  float scale_log2;           // scale * log2(e)
  int causal;
  uint64_t timeout_ns;
};

template <int DK, int DVH>
struct PrefillTraits {
  static constexpr int TILE = 128;               // q rows per CTA (MMA M)
  static constexpr int KT = 128;                 // keys per tile (MMA N of S)
  static constexpr int QCH = DK / 64;            // Q chunks ([128 x 64], 16 KB each)
  static constexpr int KCH = DK / 64;            // K chunks per key tile
  static constexpr int VCH = DVH / 64;           // V chunks per key tile (this CTA's columns)
  static constexpr int NPBUF = (DK >= 512) ? 1 : 2;
  static constexpr int RING = (DK >= 512) ? 4 : 8;
  static constexpr int SLOT = 16384;
  static constexpr int P_BYTES = 2 * SLOT;       // P: [128 x 128] as two [128 x 64] chunks
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_P = OFF_Q + QCH * SLOT;
  static constexpr int OFF_RING = OFF_P + NPBUF * P_BYTES;
  static constexpr int OFF_FLAGS = OFF_RING + RING * SLOT;   // abort, tmem base
  static constexpr int OFF_BAR = OFF_FLAGS + 16;
  // full[RING], empty[RING], q_full, s_full[2], s_free[2], p_full[NPBUF], o_done[NPBUF], drain
  static constexpr int NBAR = 2 * RING + 6 + 2 * NPBUF;
  static constexpr int SMEM_BYTES = OFF_BAR + NBAR * 8 + 1024;
  static constexpr int TMEM_S = 0;               // two S buffers, 128 columns each
  static constexpr int TMEM_O = 256;             // DVH columns
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(KCH % 2 == 0 && VCH % 2 == 0 && RING % 2 == 0, "V chunk pairs need even slots");
  static_assert(TMEM_O + DVH <= 512, "TMEM");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

template <int DK, int DVH, bool BF16>
__global__ void __launch_bounds__(192, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
  using T = PrefillTraits<DK, DVH>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);

  // Heavy-first order: the last q tiles see the most keys under the causal
  // mask, so they are handed out first; the dv parts and heads of one q tile
  // are adjacent so they read the same K/V tiles close in time.
  int64_t L = blockIdx.x;
  const int part = (int)(L % p.dv_parts);
  L /= p.dv_parts;
  const int h = (int)(L % p.Hq);
  L /= p.Hq;
  const int b = (int)(L % p.B);
  const int qt = p.n_qtiles - 1 - (int)(L / p.B);
  const int kvh = h / p.G;
  const int q0 = qt * T::TILE;
  const int skv = p.skv[b];
  const int q_last = min(q0 + T::TILE - 1, p.Sq - 1);
  int lim_last = p.causal ? q_last + skv - p.Sq + 1 : skv;  // keys visible to the last row
  lim_last = max(0, min(skv, lim_last));
  const int ntiles = (lim_last + T::KT - 1) / T::KT;

  const uint32_t qs = sbase + T::OFF_Q;
  const uint32_t ps = sbase + T::OFF_P;
  const uint32_t ring = sbase + T::OFF_RING;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + T::OFF_FLAGS);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + T::OFF_FLAGS + 4);
  const uint32_t bar0 = sbase + T::OFF_BAR;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (T::RING + s); };
  const uint32_t q_full = bar0 + 8u * (2 * T::RING);
  const uint32_t s_full = q_full + 8;                  // [2]
  const uint32_t s_free = s_full + 16;                 // [2]
  const uint32_t p_full = s_free + 16;                 // [NPBUF]
  const uint32_t o_done = p_full + 8 * T::NPBUF;       // [NPBUF]
  const uint32_t drain = o_done + 8 * T::NPBUF;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < T::RING; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full + 8 * i, 1);
      mbar_init(s_free + 8 * i, 128);
    }
    for (int i = 0; i < T::NPBUF; ++i) {
      mbar_init(p_full + 8 * i, 128);
      mbar_init(o_done + 8 * i, 1);
    }
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

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && ntiles > 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      const uint64_t pol_q = l2_policy_evict_first();
      const uint64_t pol_kv = l2_policy_evict_last();  // shared by the group's heads
      mbar_arrive_expect_tx(q_full, T::QCH * T::SLOT);
      for (int c = 0; c < T::QCH; ++c)
        tma_load_4d(qs + c * T::SLOT, &tmQ, q_full, c * 64, q0, h, b, pol_q);
      int slot = 0;
      uint32_t ph = 0;
      bool ok = true;
      auto load = [&](const CUtensorMap* map, int c0, int c1) {
        if (!ok) return;
        ok = mbar_wait(empty_bar(slot), ph ^ 1u, abort_flag, p.timeout_ns, 21);
        if (!ok) return;
        mbar_arrive_expect_tx(full_bar(slot), T::SLOT);
        tma_load_4d(ring + slot * T::SLOT, map, full_bar(slot), c0, c1, kvh, b, pol_kv);
        if (++slot == T::RING) { slot = 0; ph ^= 1u; }
      };
      for (int j = 0; j < ntiles && ok; ++j) {
        for (int c = 0; c < T::KCH; ++c) load(&tmK, c * 64, j * T::KT);
        if (j >= 1)
          for (int c = 0; c < T::VCH; ++c) load(&tmV, part * DVH + c * 64, (j - 1) * T::KT);
      }
      for (int c = 0; c < T::VCH; ++c) load(&tmV, part * DVH + c * 64, (ntiles - 1) * T::KT);
      if (!ok) {
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 2000000ull) __nanosleep(1000);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && ntiles > 0) {
      constexpr uint32_t idS = umma_idesc(128, 128, BF16, false, false);  // Q, K both K-major
      constexpr uint32_t idO = umma_idesc(128, 128, BF16, false, true);   // P K-major, V MN-major
      int slot = 0;
      uint32_t ph = 0;
      bool ok = mbar_wait(q_full, 0, abort_flag, p.timeout_ns, 22);
      tc_fence_after();
      auto pv = [&](int t) {
        if (!ok) return;
        const int pb = t % T::NPBUF;
        ok = mbar_wait(p_full + 8 * pb, (t / T::NPBUF) & 1, abort_flag, p.timeout_ns, 23);
        if (!ok) return;
        tc_fence_after();
        const uint32_t abase = ps + pb * T::P_BYTES;
        for (int i = 0; i < T::VCH / 2; ++i) {
          ok = mbar_wait(full_bar(slot), ph, abort_flag, p.timeout_ns, 24) &&
               mbar_wait(full_bar(slot + 1), ph, abort_flag, p.timeout_ns, 24);
          if (!ok) return;
          tc_fence_after();
          const uint32_t bbase = ring + slot * T::SLOT;
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            // A = P: K-major, 128-byte swizzle, keys 64*(ks/4) .. in chunk ks/4.
            const uint64_t ad =
                umma_sdesc(abase + (ks >> 2) * T::SLOT + (ks & 3) * 32, 16, 1024, SMEM_SW128);
            // B = V: MN-major (d contiguous), 128-byte swizzle; the two 64-column
            // halves are one slot apart (LBO), 8-key groups 1024 bytes (SBO).
            const uint64_t bd = umma_sdesc(bbase + ks * 2048, T::SLOT, 1024, SMEM_SW128);
            umma_ss(tmem + T::TMEM_O + i * 128, ad, bd, idO, (t > 0 || ks > 0) ? 1u : 0u);
          }
          umma_commit(empty_bar(slot));
          umma_commit(empty_bar(slot + 1));
          slot += 2;
          if (slot == T::RING) { slot = 0; ph ^= 1u; }
        }
        umma_commit(o_done + 8 * pb);
      };
      for (int j = 0; j < ntiles && ok; ++j) {
        const int sb = j & 1;
        if (j >= 2) ok = mbar_wait(s_free + 8 * sb, ((j >> 1) - 1) & 1, abort_flag, p.timeout_ns, 25);
        if (!ok) break;
        tc_fence_after();
        for (int c = 0; c < T::KCH && ok; ++c) {
          ok = mbar_wait(full_bar(slot), ph, abort_flag, p.timeout_ns, 26);
          if (!ok) break;
          tc_fence_after();
          const uint32_t bbase = ring + slot * T::SLOT;
          const uint32_t abase = qs + c * T::SLOT;
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            const uint64_t ad = umma_sdesc(abase + ks * 32, 16, 1024, SMEM_SW128);
            const uint64_t bd = umma_sdesc(bbase + ks * 32, 16, 1024, SMEM_SW128);
            umma_ss(tmem + T::TMEM_S + sb * 128, ad, bd, idS, (c > 0 || ks > 0) ? 1u : 0u);
          }
          umma_commit(empty_bar(slot));
          if (++slot == T::RING) { slot = 0; ph ^= 1u; }
        }
        if (!ok) break;
        umma_commit(s_full + 8 * sb);
        if (j >= 1) pv(j - 1);
      }
      pv(ntiles - 1);
      if (!ok) {
        umma_commit(drain);
        volatile int never = 0;
        mbar_wait(drain, 0, &never, 1000000ull, 27);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int wq = warp & 3;
    const int row = wq * 32 + lane;          // q row within the tile = TMEM lane
    const int qi = q0 + row;
    const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
    int lim = p.causal ? qi + skv - p.Sq + 1 : skv;  // keys [0, lim) visible to this row
    lim = max(0, min(skv, lim));
    volatile int own_abort = 0;
    auto wait = [&](uint32_t bar, uint32_t parity, uint32_t id) {
      return mbar_wait(bar, parity, &own_abort, p.timeout_ns, id);
    };
    float m_used = -INFINITY;  // log2-domain running max (lazily raised)
    float l = 0.f;
    bool ok = true;

    for (int j = 0; j < ntiles && ok; ++j) {
      const int sb = j & 1;
      ok = wait(s_full + 8 * sb, (j >> 1) & 1, 28);
      if (!ok) break;
      tc_fence_after();
      float s[128];
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        float tmp[16];
        tmem_ld16(tmem + lane_base + T::TMEM_S + sb * 128 + g * 16, tmp);
#pragma unroll
        for (int i = 0; i < 16; ++i) s[g * 16 + i] = tmp[i];
      }
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(s_free + 8 * sb);

      const int kb = j * T::KT;
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        const float v = (kb + c < lim) ? s[c] * p.scale_log2 : -INFINITY;
        s[c] = v;
        mx = fmaxf(mx, v);
      }
      // Raise the running max only when the tile's exceeds it by more than 8
      // (log2 units); weights stay <= 256 and O/l is unaffected.
      const bool need = mx > m_used + 8.f;
      const float m_new = need ? mx : m_used;
      const float alpha = need ? ex2(m_used - m_new) : 1.f;
      const bool warp_need = __any_sync(0xffffffffu, need);
      const int pb = j % T::NPBUF;
      if (j >= T::NPBUF) {  // P buffer pb was last read by PV(j - NPBUF)
        ok = wait(o_done + 8 * pb, ((j - T::NPBUF) / T::NPBUF) & 1, 29);
        if (!ok) break;
      }
      if (warp_need && j >= 1) {  // rescale this warp's O rows once PV(j-1) landed
        const int t = j - 1;
        ok = wait(o_done + 8 * (t % T::NPBUF), (t / T::NPBUF) & 1, 30);
        if (!ok) break;
        tc_fence_after();
#pragma unroll 1
        for (int g = 0; g < DVH / 16; ++g) {
          float o[16];
          const uint32_t ta = tmem + lane_base + T::TMEM_O + g * 16;
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

      // P row -> shared memory (K-major, 128-byte swizzle, two 64-key chunks)
      const uint32_t pbase = ps + pb * T::P_BYTES;
#pragma unroll
      for (int c8 = 0; c8 < 16; ++c8) {
        uint32_t u[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int c = c8 * 8 + 2 * e;
          const float p0 = s[c] == -INFINITY ? 0.f : ex2(s[c] - m_used);
          const float p1 = s[c + 1] == -INFINITY ? 0.f : ex2(s[c + 1] - m_used);
          u[e] = pack2(p0, p1, BF16);
          l += p0 + p1;
        }
        st_shared_v4(pbase + (c8 >> 3) * T::SLOT + sw128_offset(row, (c8 & 7) * 8), u[0], u[1],
                     u[2], u[3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full + 8 * pb);
    }

    // ---------------------------------------------------------- epilogue
    if (ok && ntiles > 0) {
      const int t = ntiles - 1;
      ok = wait(o_done + 8 * (t % T::NPBUF), (t / T::NPBUF) & 1, 31);
      if (ok) tc_fence_after();
    }
    if (ok) {
      const float inv = l > 0.f ? 1.f / l : 0.f;
      uint8_t* orow = reinterpret_cast<uint8_t*>(p.out) +
                      ((int64_t)b * p.o_sb + (int64_t)h * p.o_sh + (int64_t)qi * p.o_ss +
                       part * DVH) * 2;
#pragma unroll 1
      for (int g = 0; g < DVH / 16; ++g) {
        float o[16];
        if (ntiles > 0) {
          tmem_ld16(tmem + lane_base + T::TMEM_O + g * 16, o);
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
      if (part == 0 && p.lse && qi < p.Sq)
        p.lse[((int64_t)b * p.Hq + h) * p.Sq + qi] =
            l > 0.f ? (m_used + __log2f(l)) * 0.69314718055994531f : -INFINITY;
    }
    if (!ok) *abort_flag = 1;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, T::TMEM_COLS);
  }
}

}  // namespace attn
