// decode_kernel.cuh -- split-KV decode (one query row per head, Sq == 1).
//
// Decode reads the whole KV cache once per step and is bandwidth-bound
// ("GQA和MLA详解" section 1; "Full 路线" section 4.5).  Every KV byte must
// therefore be read from HBM once for all G query heads that share it
// ("GQA和MLA详解" section 2: real kernels index the shared head instead of
// copying it).  This kernel puts 128 keys of one KV head in the MMA M
// dimension and the group's query heads in N ("keys x heads" orientation):
//
//   S^T[128 keys x NH heads] = K_tile[128 x d_k] * Q^T          (tcgen05, TMEM)
//   softmax over keys per head (online, with a lazily updated max)
//   O^T[d_v x NH]           += V_tile^T[d_v x 128] * P^T[128 x NH]
//
// so G = 16 MQA heads, G = 8 GQA heads (padded to 16) and 64 of the 128 MLA
// heads are MMA-efficient without padding M.  Each CTA handles one
// (batch, kv head, head block, KV split); partial outputs (normalised) and
// their LSEs go to the workspace and a combine kernel merges the splits.
//
// MLA absorbed mode ("Full 路线" sections 4.2-4.3): K rows are the cached
// [c_kv | k_pe] rows (d_k = 576) and V is the first 512 columns of the same
// rows (d_v = 512), read through a second tensor map over the same memory.
//
// Warp roles (192 threads): warp 0 issues TMA loads, warp 1 allocates TMEM
// and issues UMMA, warps 2-5 run the softmax (thread = key row of the tile;
// for O^T, thread = d_v row of each 128-row block) and the epilogue.
#pragma once

#include "sm100.cuh"

namespace attn {

struct DecodeParams {
  const void* q;         // [B, Hq, 1, d_k]
  int64_t q_sb, q_sh;    // element strides of q
  const int32_t* skv;    // [B] keys per sequence (device)
  float* ws_o;           // [B, Hq, num_splits, d_v] normalised partial outputs
  float* ws_lse;         // [B, Hq, num_splits] partial LSE (natural log)
  int B, Hq, Hkv, G;
  int num_splits, split_tiles, head_blocks;
  float scale_log2;      // scale * log2(e)
  uint64_t timeout_ns;
};

constexpr uint32_t ceil_pow2_cols(uint32_t n) {
  uint32_t c = 32;
  while (c < n) c <<= 1;
  return c;
}

template <int DK, int DV, int NH>
struct DecodeTraits {
  static constexpr int TILE = 128;                 // keys per tile (MMA M)
  static constexpr int KCH = DK / 64;              // 64-column K chunks per tile
  static constexpr int KSLOTS = (KCH + 1) & ~1;    // ring slots per tile's K (even)
  static constexpr int VCH = DV / 64;              // 64-column V chunks per tile
  static constexpr int DVB = DV / 128;             // 128-row blocks of O^T
  static constexpr int RING = (DK == 576) ? 6 : (DK == 512 ? 4 : 6);
  static constexpr int MIN_CTAS = (DK == 576) ? 1 : 2;
  static constexpr int SLOT = 16384;               // one [128 x 64] 2-byte chunk
  static constexpr int QT_CHUNK = NH * 128;        // one [NH x 64] chunk of Q^T
  static constexpr int PT_BYTES = NH * TILE * 2;   // one P^T buffer
  static constexpr int OFF_RING = 0;
  static constexpr int OFF_QT = OFF_RING + RING * SLOT;
  static constexpr int OFF_PT = OFF_QT + KCH * QT_CHUNK;
  static constexpr int OFF_RED = OFF_PT + 2 * PT_BYTES;         // float [2][4][NH]
  static constexpr int OFF_M = OFF_RED + 2 * 4 * NH * 4;        // float [NH] running max
  static constexpr int OFF_ALPHA = OFF_M + NH * 4;              // float [NH] rescale factors
  static constexpr int OFF_L = OFF_ALPHA + NH * 4;              // float [NH] final sums
  static constexpr int OFF_FLAGS = OFF_L + NH * 4;              // int [4]: any[2], abort, tmem
  static constexpr int OFF_BAR = (OFF_FLAGS + 16 + 7) & ~7;
  // barriers: full[RING], empty[RING], s_full[2], s_free[2], p_full[2], o_done[2], q_full,
  // red_full[2], stat_ready[2], drain
  static constexpr int NBAR = 2 * RING + 14;
  static constexpr int SMEM_BYTES = OFF_BAR + NBAR * 8 + 1024;  // + alignment slack
  static constexpr int TMEM_S = 0;                  // S^T double buffer: 2 x NH columns
  static constexpr int TMEM_O = 2 * NH;             // O^T: DVB x NH columns
  static constexpr uint32_t TMEM_COLS = ceil_pow2_cols(2 * NH + DVB * NH);
  static_assert(KCH * QT_CHUNK % 1024 == 0, "Q^T chunks must keep 1024-byte alignment");
  static_assert(RING % 2 == 0 && KSLOTS % 2 == 0 && VCH % 2 == 0, "V chunk pairs need even slots");
  static_assert(NH % 16 == 0 && NH <= 256, "MMA N");
  static_assert(TMEM_COLS <= 512, "TMEM");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

template <int DK, int DV, int NH, bool BF16>
__global__ void __launch_bounds__(192, DecodeTraits<DK, DV, NH>::MIN_CTAS)
    decode_split_kernel(const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const DecodeParams p) {
  using T = DecodeTraits<DK, DV, NH>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);

  const int hb = blockIdx.x % p.head_blocks;
  const int split = blockIdx.x / p.head_blocks;
  const int b = blockIdx.y;
  const int kvh = blockIdx.z;
  const int skv = p.skv[b];
  const int tok_begin = split * p.split_tiles * T::TILE;
  if (tok_begin >= skv) return;  // nothing of this sequence in this split (uniform)
  const int tok_end = min(skv, tok_begin + p.split_tiles * T::TILE);
  const int ntiles = (tok_end - tok_begin + T::TILE - 1) / T::TILE;
  const int h0 = kvh * p.G + hb * NH;            // first query head of this CTA
  const int nvalid = min(NH, p.G - hb * NH);     // real heads among the NH rows

  const uint32_t ring = sbase + T::OFF_RING;
  const uint32_t qt = sbase + T::OFF_QT;
  const uint32_t pt = sbase + T::OFF_PT;
  float* red = reinterpret_cast<float*>(smem + T::OFF_RED);
  float* m_sm = reinterpret_cast<float*>(smem + T::OFF_M);
  float* alpha_sm = reinterpret_cast<float*>(smem + T::OFF_ALPHA);
  float* l_sm = reinterpret_cast<float*>(smem + T::OFF_L);
  volatile int* flags = reinterpret_cast<volatile int*>(smem + T::OFF_FLAGS);
  volatile int* abort_flag = flags + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + T::OFF_FLAGS + 12);
  const uint32_t bar0 = sbase + T::OFF_BAR;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (T::RING + s); };
  const uint32_t s_full = bar0 + 8u * (2 * T::RING);      // [2]
  const uint32_t s_free = s_full + 16;                    // [2]
  const uint32_t p_full = s_free + 16;                    // [2]
  const uint32_t o_done = p_full + 16;                    // [2]
  const uint32_t q_full = o_done + 16;
  const uint32_t red_full = q_full + 8;                   // [2]
  const uint32_t stat_ready = red_full + 16;              // [2]
  const uint32_t drain = stat_ready + 16;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < T::RING; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full + 8 * i, 1);
      mbar_init(s_free + 8 * i, 128);
      mbar_init(p_full + 8 * i, 128);
      mbar_init(o_done + 8 * i, 1);
    }
    mbar_init(q_full, 128);
    for (int i = 0; i < 2; ++i) {
      mbar_init(red_full + 8 * i, 128);
      mbar_init(stat_ready + 8 * i, NH);
    }
    mbar_init(drain, 1);
    flags[0] = 0;
    flags[1] = 0;
    flags[2] = 0;
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
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      const uint64_t pol = l2_policy_evict_first();
      int slot = 0;
      uint32_t ph = 0;
      bool ok = true;
      auto load = [&](const CUtensorMap* map, int c0, int c1) {
        if (!ok) return;
        ok = mbar_wait(empty_bar(slot), ph ^ 1u, abort_flag, p.timeout_ns, 1);
        if (!ok) return;
        mbar_arrive_expect_tx(full_bar(slot), T::SLOT);
        tma_load_4d(ring + slot * T::SLOT, map, full_bar(slot), c0, c1, kvh, b, pol);
        if (++slot == T::RING) { slot = 0; ph ^= 1u; }
      };
      auto phantom = [&]() {
        if (!ok) return;
        ok = mbar_wait(empty_bar(slot), ph ^ 1u, abort_flag, p.timeout_ns, 2);
        if (!ok) return;
        mbar_arrive(full_bar(slot));
        if (++slot == T::RING) { slot = 0; ph ^= 1u; }
      };
      for (int j = 0; j < ntiles && ok; ++j) {
        const int t0 = tok_begin + j * T::TILE;
        for (int c = 0; c < T::KCH; ++c) load(&tmK, c * 64, t0);
        if (T::KSLOTS > T::KCH) phantom();
        if (j >= 1)
          for (int c = 0; c < T::VCH; ++c) load(&tmV, c * 64, t0 - T::TILE);
      }
      {
        const int t0 = tok_begin + (ntiles - 1) * T::TILE;
        for (int c = 0; c < T::VCH; ++c) load(&tmV, c * 64, t0);
      }
      // On abort, give every copy this thread started time to land before
      // the CTA leaves (a tile copy takes microseconds; wait 2 ms).
      if (!ok) {
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 2000000ull) __nanosleep(1000);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = umma_idesc(128, NH, BF16, false, false);
      constexpr uint32_t idO = umma_idesc(128, NH, BF16, true, true);
      int slot = 0;
      uint32_t ph = 0;
      bool ok = mbar_wait(q_full, 0, abort_flag, p.timeout_ns, 3);
      tc_fence_after();
      auto pv = [&](int t) {
        if (!ok) return;
        const int pb = t & 1;
        ok = mbar_wait(p_full + 8 * pb, (t >> 1) & 1, abort_flag, p.timeout_ns, 4);
        if (!ok) return;
        tc_fence_after();
        const uint32_t bbase = pt + pb * T::PT_BYTES;
        for (int i = 0; i < T::DVB; ++i) {
          ok = mbar_wait(full_bar(slot), ph, abort_flag, p.timeout_ns, 5) &&
               mbar_wait(full_bar(slot + 1), ph, abort_flag, p.timeout_ns, 5);
          if (!ok) return;
          tc_fence_after();
          const uint32_t abase = ring + slot * T::SLOT;
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            // A = V^T: MN-major, 128-byte swizzle; the two 64-row halves of
            // the 128-row block sit one slot apart (LBO); 8-key groups are
            // 1024 bytes apart (SBO); 16 keys per K step = 2048 bytes.
            const uint64_t ad = umma_sdesc(abase + ks * 2048, T::SLOT, 1024, SMEM_SW128);
            // B = P^T: MN-major, no swizzle; 8x8 core matrices, 8-head groups
            // 128 bytes apart (SBO), 8-key groups NH*16 bytes apart (LBO).
            const uint64_t bd = umma_sdesc(bbase + ks * 2 * NH * 16, NH * 16, 128, SMEM_NOSWIZZLE);
            umma_ss(tmem + T::TMEM_O + i * NH, ad, bd, idO, (t > 0 || ks > 0) ? 1u : 0u);
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
        if (j >= 2) ok = mbar_wait(s_free + 8 * sb, ((j >> 1) - 1) & 1, abort_flag, p.timeout_ns, 6);
        if (!ok) break;
        tc_fence_after();
        for (int c = 0; c < T::KCH && ok; ++c) {
          ok = mbar_wait(full_bar(slot), ph, abort_flag, p.timeout_ns, 7);
          if (!ok) break;
          tc_fence_after();
          const uint32_t abase = ring + slot * T::SLOT;
          const uint32_t bbase = qt + c * T::QT_CHUNK;
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            // A = K tile, B = Q^T: both K-major, 128-byte swizzle, 8-row
            // groups 1024 bytes apart; 16 columns per K step = 32 bytes.
            const uint64_t ad = umma_sdesc(abase + ks * 32, 16, 1024, SMEM_SW128);
            const uint64_t bd = umma_sdesc(bbase + ks * 32, 16, 1024, SMEM_SW128);
            umma_ss(tmem + T::TMEM_S + sb * NH, ad, bd, idS, (c > 0 || ks > 0) ? 1u : 0u);
          }
          umma_commit(empty_bar(slot));
          if (++slot == T::RING) { slot = 0; ph ^= 1u; }
        }
        if (ok && T::KSLOTS > T::KCH) {
          ok = mbar_wait(full_bar(slot), ph, abort_flag, p.timeout_ns, 8);
          if (ok) {
            mbar_arrive(empty_bar(slot));
            if (++slot == T::RING) { slot = 0; ph ^= 1u; }
          }
        }
        if (!ok) break;
        umma_commit(s_full + 8 * sb);
        if (j >= 1) pv(j - 1);
      }
      pv(ntiles - 1);
      if (!ok) {
        // Gave up: let every MMA already issued finish before TMEM is freed.
        umma_commit(drain);
        volatile int never = 0;
        mbar_wait(drain, 0, &never, 1000000ull, 13);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax
    // Cross-warp exchanges use mbarriers with bounded waits (red_full: all
    // 128 partial maxima written; stat_ready: the per-head maxima, rescale
    // factors and the "any head rescaled" flag published), so that a wait
    // that gives up can never leave the other warps parked on a barrier.
    // These threads do not consult the abort flag: all 128 wait on the same
    // barriers, so they either all see a barrier complete or all time out.
    const int st = threadIdx.x - 64;       // 0..127
    const int wq = warp & 3;               // TMEM lane quarter of this warp
    const int row = wq * 32 + lane;        // key row of S^T / d_v row of O^T blocks
    const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
    volatile int own_abort = 0;
    auto wait = [&](uint32_t bar, uint32_t parity, uint32_t id) {
      return mbar_wait(bar, parity, &own_abort, p.timeout_ns, id);
    };

    // Q^T -> shared memory, K-major 128-byte-swizzled [NH x 64] chunks;
    // rows past the group's heads are zero.
    {
      const uint8_t* qg = reinterpret_cast<const uint8_t*>(p.q);
      constexpr int PIECES_PER_ROW = DK / 8;  // 16-byte pieces
      for (int idx = st; idx < NH * PIECES_PER_ROW; idx += 128) {
        const int r = idx / PIECES_PER_ROW;
        const int col = (idx % PIECES_PER_ROW) * 8;
        uint4 val = make_uint4(0u, 0u, 0u, 0u);
        if (r < nvalid) {
          const int64_t off = (int64_t)b * p.q_sb + (int64_t)(h0 + r) * p.q_sh + col;
          val = __ldg(reinterpret_cast<const uint4*>(qg + off * 2));
        }
        st_shared_v4(qt + (col / 64) * T::QT_CHUNK + sw128_offset(r, col % 64), val.x, val.y,
                     val.z, val.w);
      }
      if (st < NH) m_sm[st] = -INFINITY;
      fence_proxy_async_smem();
      mbar_arrive(q_full);
      named_bar_sync(1, 128);  // m_sm initialised before anyone reads it
    }

    float l[NH];
#pragma unroll
    for (int h = 0; h < NH; ++h) l[h] = 0.f;
    bool ok = true;

    for (int j = 0; j < ntiles && ok; ++j) {
      const int sb = j & 1;
      const uint32_t par = (j >> 1) & 1;
      ok = wait(s_full + 8 * sb, par, 9);
      if (!ok) break;
      tc_fence_after();
      float s[NH];
#pragma unroll
      for (int g = 0; g < NH / 16; ++g) {
        float tmp[16];
        tmem_ld16(tmem + lane_base + T::TMEM_S + sb * NH + g * 16, tmp);
#pragma unroll
        for (int i = 0; i < 16; ++i) s[g * 16 + i] = tmp[i];
      }
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(s_free + 8 * sb);

      // per-head maximum over the tile's 128 keys
      const bool valid = tok_begin + j * T::TILE + row < tok_end;
      float* rbuf = red + sb * 4 * NH;
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        float v = valid ? s[h] * p.scale_log2 : -INFINITY;
        s[h] = v;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
        if (lane == 0) rbuf[wq * NH + h] = v;
      }
      mbar_arrive(red_full + 8 * sb);
      ok = wait(red_full + 8 * sb, par, 14);
      if (!ok) break;
      if (st == 0) flags[sb ^ 1] = 0;
      if (st < NH) {
        const float tm = fmaxf(fmaxf(rbuf[st], rbuf[NH + st]), fmaxf(rbuf[2 * NH + st], rbuf[3 * NH + st]));
        const float mo = m_sm[st];
        // Keep the stale maximum unless the tile's exceeds it by more than
        // 8 (log2 units): exp2(s - m) then stays <= 256, and the final
        // division by the sum accumulated against the same maximum is exact.
        const bool need = tm > mo + 8.f;
        const float mn = need ? tm : mo;
        alpha_sm[st] = need ? ex2(mo - mn) : 1.f;
        m_sm[st] = mn;
        if (need) flags[sb] = 1;
        mbar_arrive(stat_ready + 8 * sb);
      }
      ok = wait(stat_ready + 8 * sb, par, 15);
      if (!ok) break;
      const bool any = flags[sb] != 0;

      if (j >= 2) {  // P^T buffer sb was last read by PV(j-2)
        ok = wait(o_done + 8 * sb, ((j - 2) >> 1) & 1, 10);
        if (!ok) break;
      }
      if (any && j >= 1) {  // rescale O^T once PV(j-1) has landed
        ok = wait(o_done + 8 * ((j - 1) & 1), ((j - 1) >> 1) & 1, 11);
        if (!ok) break;
        tc_fence_after();
#pragma unroll 1
        for (int i = 0; i < T::DVB; ++i) {
#pragma unroll
          for (int g = 0; g < NH / 16; ++g) {
            float o[16];
            const uint32_t ta = tmem + lane_base + T::TMEM_O + i * NH + g * 16;
            tmem_ld16(ta, o);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 16; ++c) o[c] *= alpha_sm[g * 16 + c];
            tmem_st16(ta, o);
          }
        }
        tmem_wait_st();
      }
#pragma unroll
      for (int h = 0; h < NH; ++h) l[h] *= alpha_sm[h];

      // P^T row for this key: NH values, written as MN-major core matrices.
      const uint32_t prow = pt + sb * T::PT_BYTES + (row >> 3) * (NH * 16) + (row & 7) * 16;
#pragma unroll
      for (int g = 0; g < NH / 8; ++g) {
        uint32_t u[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int h = g * 8 + 2 * e;
          const float p0 = s[h] == -INFINITY ? 0.f : ex2(s[h] - m_sm[h]);
          const float p1 = s[h + 1] == -INFINITY ? 0.f : ex2(s[h + 1] - m_sm[h + 1]);
          u[e] = pack2(p0, p1, BF16);
          l[h] += p0;
          l[h + 1] += p1;
        }
        st_shared_v4(prow + g * 128, u[0], u[1], u[2], u[3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full + 8 * sb);
    }

    // ---------------------------------------------------------- epilogue
    if (ok) {
      const int last = ntiles - 1;
      ok = wait(o_done + 8 * (last & 1), (last >> 1) & 1, 12);
    }
    if (ok) {
      tc_fence_after();
      // the reduction buffers and barriers continue their per-tile sequence
      const int sb = ntiles & 1;
      const uint32_t par = (ntiles >> 1) & 1;
      float* rbuf = red + sb * 4 * NH;
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        float v = l[h];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) rbuf[wq * NH + h] = v;
      }
      mbar_arrive(red_full + 8 * sb);
      ok = wait(red_full + 8 * sb, par, 16);
      if (ok && st < NH) {
        const float L = (rbuf[st] + rbuf[NH + st]) + (rbuf[2 * NH + st] + rbuf[3 * NH + st]);
        l_sm[st] = L;
        if (st < nvalid) {
          const int64_t idx = ((int64_t)b * p.Hq + h0 + st) * p.num_splits + split;
          p.ws_lse[idx] = L > 0.f ? (m_sm[st] + __log2f(L)) * 0.69314718055994531f : -INFINITY;
        }
        mbar_arrive(stat_ready + 8 * sb);
      }
      if (ok) ok = wait(stat_ready + 8 * sb, par, 17);
    }
    if (ok) {
#pragma unroll 1
      for (int i = 0; i < T::DVB; ++i) {
#pragma unroll
        for (int g = 0; g < NH / 16; ++g) {
          float o[16];
          tmem_ld16(tmem + lane_base + T::TMEM_O + i * NH + g * 16, o);
          tmem_wait_ld();
          const int d = i * 128 + row;
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int h = g * 16 + c;
            if (h < nvalid) {
              const float L = l_sm[h];
              const int64_t idx = (((int64_t)b * p.Hq + h0 + h) * p.num_splits + split) * DV + d;
              p.ws_o[idx] = L > 0.f ? o[c] / L : 0.f;
            }
          }
        }
      }
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

// ---------------------------------------------------------------- combine
//
// out[b,h,0,:] = sum_s exp(lse_s - L) o_s,  L = log sum_s exp(lse_s), over
// the splits that hold keys of sequence b, in split order (no atomics, so
// the result is bitwise reproducible: "GQA和MLA详解" section 4 on reduction
// order).
struct CombineParams {
  const float* ws_o;
  const float* ws_lse;
  const int32_t* skv;
  void* out;
  int64_t o_sb, o_sh;
  float* lse;  // [B, Hq] (Sq == 1) or NULL
  int B, Hq, DV, num_splits, split_tokens;
};

template <bool BF16>
__global__ void __launch_bounds__(128) combine_kernel(const CombineParams p) {
  const int bh = blockIdx.x;
  const int b = bh / p.Hq;
  const int h = bh % p.Hq;
  const int skv = p.skv[b];
  const int n = min(p.num_splits, (skv + p.split_tokens - 1) / p.split_tokens);
  const float* lse_s = p.ws_lse + (int64_t)bh * p.num_splits;
  float mx = -INFINITY;
  for (int s = 0; s < n; ++s) mx = fmaxf(mx, lse_s[s]);
  float L = -INFINITY;
  if (n > 0 && mx != -INFINITY) {
    float acc = 0.f;
    for (int s = 0; s < n; ++s) acc += __expf(lse_s[s] - mx);
    L = mx + __logf(acc);
  }
  const float* o_s = p.ws_o + (int64_t)bh * p.num_splits * p.DV;
  uint8_t* outp = reinterpret_cast<uint8_t*>(p.out) + ((int64_t)b * p.o_sb + (int64_t)h * p.o_sh) * 2;
  for (int d = threadIdx.x * 2; d < p.DV; d += 256) {
    float a0 = 0.f, a1 = 0.f;
    if (L != -INFINITY) {
      for (int s = 0; s < n; ++s) {
        const float w = __expf(lse_s[s] - L);
        const float2 v = *reinterpret_cast<const float2*>(o_s + (int64_t)s * p.DV + d);
        a0 = fmaf(w, v.x, a0);
        a1 = fmaf(w, v.y, a1);
      }
    }
    *reinterpret_cast<uint32_t*>(outp + (int64_t)d * 2) = pack2(a0, a1, BF16);
  }
  if (threadIdx.x == 0 && p.lse) p.lse[bh] = L;
}

}  // namespace attn
