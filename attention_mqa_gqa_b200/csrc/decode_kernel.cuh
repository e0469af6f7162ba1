// decode_kernel.cuh -- persistent split-KV decode: one query per head
// (Sq == 1), or a few (Sq = 2..16, a power of two: extend / speculative
// verification) against the KV cache, head dim 128 or 512.
//
// Decode reads the whole KV cache once per step and is bandwidth-bound
// ("GQA和MLA详解" section 1; "Full 路线" section 4.5), so every K/V byte
// must be read from HBM once for all G query heads that share it
// ("GQA和MLA详解" section 2: real kernels index the shared head instead of
// copying it).  This kernel puts 128 keys of one KV head in the MMA M
// dimension and NH = 16 columns in N, a column being one (query head,
// query) pair of the group:
//
//   S^T[128 keys x NH] = K_tile[128 x d_k] * Q^T                 (tcgen05, TMEM)
//   softmax over keys per column (online, with a lazily raised max)
//   O^T[d_v x NH]     += V_tile^T[d_v x 128] * P^T[128 x NH]
//
// so the 16 heads of MQA, or the 8 heads of a GQA group (N padded to 16, or
// filled by 8 heads x 2 queries), use the tensor cores without padding the
// 128-row M dimension with absent query rows.  With Sq > 1 each column
// carries its own bottom-right causal limit.
//
// Scheduling: the grid is persistent (one wave).  The key tiles of all
// (sequence, kv head) units, laid end to end, are cut into `ranges` equal
// contiguous ranges; each CTA (with one CTA per head block of the group)
// walks its range, which may span several units.  Each maximal piece of a
// unit inside a range produces one normalised partial output and its LSE
// in slot (range + unit) of the workspace; combine_kernel.cuh merges the
// pieces of each unit in range order.  Every SM gets the same number of
// key tiles whatever the mix of sequence lengths.  A sequence's partial
// last tile is read as the 128 rows ending at its last key, so no cache row
// past the sequence is ever read.
//
// The absorbed-MLA rows (d_k = 576, V = their first 512 columns) run on
// SM pairs in mla_pair_kernel.cuh, which reuses the scheduling here.
//
// Warp roles (320 threads): warp 0 lane 0 streams K/V chunks through the
// ring and lane 1 loads Q^T per piece (both TMA), warp 1 allocates TMEM and
// issues UMMA, warps 2-9 run the softmax and the epilogues: two threads per
// key row of the tile (for O^T, per d_v row of each 128-row block), each
// owning half of the group's heads.
#pragma once

#include "sm100.cuh"

namespace attn {

struct DecodeParams {
  const int32_t* skv;    // [B] keys per sequence (device)
  float* ws_o;           // [ranges + B*Hkv][G*Sq][d_v] normalised partial outputs
  float* ws_lse;         // [ranges + B*Hkv][G*Sq] partial LSE (natural log)
  int B, Hq, Hkv, G;
  int Sq;                // queries per sequence (1, or a few for extend / speculative decode)
  int causal;            // Sq > 1: query i sees keys j <= i + skv[b] - Sq
  int ranges, head_blocks;
  float scale_log2;      // scale * log2(e)
  uint64_t timeout_ns;
  // In-kernel merge (attn_fwd): the last CTA to finish a piece of a unit
  // merges the unit's pieces into `out` / `lse`.  `counters` (one per unit
  // and head block, per CTA of a pair for the MLA kernel) are zeroed by
  // decode_prepare_kernel just before.  counters == nullptr leaves the merge
  // to combine_kernel (attn_decode_partial, then attn_decode_combine).
  unsigned int* counters;
  void* out;                  // [B, Hq, Sq, d_v]
  int64_t o_sb, o_sh, o_ss;   // element strides of out
  float* lse;                 // [B, Hq, Sq] or NULL
  // Top-k MLA decode with the rows gathered inside the kernel: key j of
  // sequence b is row idx[b * idx_sb + j] of the latent cache `src` (one
  // kv head), j < skv[b]; a position outside [0, src_len[b]) reads as a
  // zero row and sets bit 2 of the device error word.
  const int32_t* idx;
  int64_t idx_sb;
  const uint8_t* src;         // byte address of the cache
  int64_t src_sb, src_ss;     // element strides of the cache (sequence, row)
  const int32_t* src_len;     // [B] valid cache rows per sequence
};

constexpr uint32_t ceil_pow2_cols(uint32_t n) {
  uint32_t c = 32;
  while (c < n) c <<= 1;
  return c;
}

// Key tiles of a sequence: tiles of 2^shift keys (128 for one CTA, 256 for
// a CTA pair).
__device__ __forceinline__ int key_tiles(int skv, int shift) {
  return (skv + (1 << shift) - 1) >> shift;
}

template <int DK, int DV, int NH>
struct DecodeTraits {
  static constexpr int TILE = 128;                 // keys per tile (MMA M)
  static constexpr int KCH = DK / 64;              // 64-column K chunks per tile
  static constexpr int VCH = DV / 64;              // 64-column V chunks per tile
  // One TMA copy moves GCH consecutive chunks of a tile into one ring group
  // (a single copy of 16 KB per chunk caps a CTA's stream well below HBM
  // bandwidth).  With an odd chunk count the last K group's second chunk
  // lies past the row's end and is zero-filled by the copy.
  static constexpr int GCH = 2;
  static constexpr int KG = (KCH + GCH - 1) / GCH;  // ring groups per K tile
  static constexpr int VG = VCH / GCH;              // ring groups per V tile (one per O^T block)
  static constexpr int DVB = DV / 128;             // 128-row blocks of O^T
  // resident CTAs per SM: at d = 512 one CTA per SM with a deeper ring
  // (with ~8 key tiles per range instead of ~4 the tiles split more evenly
  // over the ranges); at d = 128 two
  static constexpr int CTAS = (DK == 128) ? 2 : 1;
  static constexpr int RING = (DK == 512) ? 8 : 6;
  static constexpr int NPT = 2;                    // P^T buffers
  static constexpr int SOFTMAX_THREADS = 256;      // two threads per key row
  static constexpr int THREADS = 64 + SOFTMAX_THREADS;
  static constexpr int NQ = (DK == 512) ? 2 : 1;   // Q^T buffers (next piece's Q^T prefetched)
  static constexpr int SLOT = 16384;               // one [128 x 64] 2-byte chunk
  static constexpr int GBYTES = GCH * SLOT;         // one ring group
  static constexpr int RING_G = RING / GCH;         // ring groups
  static constexpr int QT_CHUNK = NH * 128;        // one [NH x 64] chunk of Q^T
  static constexpr int PT_BYTES = NH * TILE * 2;   // one P^T buffer
  static constexpr int OFF_RING = 0;
  static constexpr int OFF_QT = OFF_RING + RING * SLOT;
  static constexpr int QT_BYTES = KCH * QT_CHUNK;   // one Q^T buffer
  static constexpr int OFF_PT = OFF_QT + NQ * QT_BYTES;
  static constexpr int OFF_RED = OFF_PT + NPT * PT_BYTES;       // float [2][4][NH]
  static constexpr int OFF_M = OFF_RED + 2 * 4 * NH * 4;        // float [NH] running max
  static constexpr int OFF_ALPHA = OFF_M + NH * 4;              // float [NH] rescale factors
  static constexpr int OFF_L = OFF_ALPHA + NH * 4;              // float [NH] final sums
  static constexpr int OFF_SCAN = OFF_L + NH * 4;               // int64 [8] block scan
  static constexpr int OFF_SCHED = OFF_SCAN + 64;               // int [4] range start
  static constexpr int OFF_POS = OFF_SCHED + 16;                // int64 [4] range position
  static constexpr int OFF_FLAGS = OFF_POS + 32;                // int [4]: any[2], abort, tmem
  static constexpr int OFF_MERGE = OFF_FLAGS + 16;              // int: this CTA merges a unit
  static constexpr int OFF_BAR = (OFF_MERGE + 16 + 7) & ~7;
  // full[RING_G], empty[RING_G], s_full[2], s_free[2], p_full[NPT], o_done[NPT], q_full[NQ],
  // q_free[NQ], red_full[2], stat_ready[2], drain
  static constexpr int NBAR = 2 * RING_G + 11 + 2 * NPT + 2 * NQ;
  static constexpr int SMEM_BYTES = OFF_BAR + NBAR * 8 + 1024;  // + alignment slack
  static constexpr int TMEM_S = 0;                  // S^T double buffer: 2 x NH columns
  static constexpr int TMEM_O = 2 * NH;             // O^T: DVB x NH columns
  static constexpr uint32_t TMEM_COLS = ceil_pow2_cols(2 * NH + DVB * NH);
  static_assert(QT_BYTES % 1024 == 0, "Q^T buffers must keep 1024-byte alignment");
  static_assert(OFF_PT % 1024 == 0, "P^T alignment");
  static_assert(GCH == 2 && RING % GCH == 0 && VG == DVB, "a V group is one 128-row O^T block");
  static_assert(NH % 16 == 0 && NH <= 256, "MMA N");
  static_assert(TMEM_COLS * CTAS <= 512, "TMEM");
  static_assert(SMEM_BYTES * CTAS <= 232448, "shared memory");
};

// Maximum over the 32 lanes of a warp for each of NH values per lane, as a
// transposed butterfly: at each exchange distance a lane keeps half of its
// live values (the half its lane bit selects), swaps the other half with
// its partner and keeps the maxima, so NH/2 + NH/4 + ... shuffles replace
// 5 * NH.  Afterwards lane l holds in v[0 .. max(NH/32, 1) - 1] the maxima of
// heads transposed_head<NH>(l, i).
template <int NH, int N, int OFF>
__device__ __forceinline__ void transposed_warp_max(float (&v)[NH], int lane) {
  if constexpr (OFF > 0) {
    if constexpr (N == 1) {
      v[0] = fmaxf(v[0], __shfl_xor_sync(0xffffffffu, v[0], OFF));
      transposed_warp_max<NH, 1, OFF / 2>(v, lane);
    } else {
      constexpr int H = N / 2;
      const bool upper = (lane & OFF) != 0;
#pragma unroll
      for (int i = 0; i < H; ++i) {
        const float keep = upper ? v[i + H] : v[i];
        const float send = upper ? v[i] : v[i + H];
        v[i] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, OFF));
      }
      transposed_warp_max<NH, H, OFF / 2>(v, lane);
    }
  }
}

template <int NH>
__device__ __forceinline__ int transposed_head(int lane, int i) {
  if constexpr (NH >= 32) return lane * (NH / 32) + i;
  else return lane / (32 / NH);
}

// Walks the pieces of one key range: consecutive (sequence b, kv head) units
// in b-major order, each piece covering tiles [tile0, tile0 + ntiles) of one
// unit.  Every role of the CTA runs its own copy over the same range.
struct PieceWalker {
  const int32_t* skv;
  int B, Hkv, shift;
  int b, kvh, off, remaining;
  long long gpos = 0;  // global index (over all units' tiles) of the next piece's first tile

  __device__ bool next(int& pb, int& pkvh, int& tile0, int& ntiles) {
    long long g;
    return next(pb, pkvh, tile0, ntiles, g);
  }
  __device__ bool next(int& pb, int& pkvh, int& tile0, int& ntiles, long long& gstart) {
    if (remaining <= 0) return false;
    const int tb = key_tiles(skv[b], shift);
    const int n = min(remaining, tb - off);
    pb = b;
    pkvh = kvh;
    tile0 = off;
    ntiles = n;
    gstart = gpos;
    gpos += n;
    remaining -= n;
    off = 0;
    if (remaining > 0) {
      if (++kvh == Hkv) {
        kvh = 0;
        do { ++b; } while (b < B && key_tiles(skv[b], shift) == 0);
      }
    }
    return true;
  }
};

// Range `r` of min(R, T) equal ranges over the T concatenated key tiles of
// all units (unit u = b * Hkv + kvh holds ceil(skv[b] / 128) tiles).  Called
// by all threads of the CTA; leaves the range's first unit, tile offset and
// length in sched[0..3] (length 0: no range r), and in pos[0..2] the range's
// first global tile, T and the number of ranges in use.
__device__ __forceinline__ void locate_range(const int32_t* skv, int B, int Hkv, int shift, int R,
                                             int r, long long* scan, int* sched, long long* pos) {
  const int tid = threadIdx.x;
  const int nt = blockDim.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int c = (B + nt - 1) / nt;
  const int lo = min(B, tid * c), hi = min(B, lo + c);
  long long mine = 0;
  for (int b = lo; b < hi; ++b) mine += key_tiles(skv[b], shift);
  long long v = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) scan[warp] = v;
  __syncthreads();
  long long before = 0, total = 0;
  for (int w = 0; w < (nt >> 5); ++w) {
    if (w < warp) before += scan[w];
    total += scan[w];
  }
  const long long T = total * Hkv;
  // With fewer tiles than ranges only the first T ranges are used, so that
  // every range in use holds at least one tile (the combine relies on it).
  const long long Re = T < R ? T : R;
  const long long x0 = r < Re ? (long long)r * T / Re : T;
  const long long x1 = r < Re ? (long long)(r + 1) * T / Re : T;
  if (tid == 0) {
    sched[3] = (int)(x1 - x0);
    pos[0] = x0;
    pos[1] = T;
    pos[2] = Re;
  }
  long long run = before + v - mine;  // tiles of sequences before `lo`
  for (int b = lo; b < hi; ++b) {
    const int tb = key_tiles(skv[b], shift);
    const long long base = run * Hkv;
    if (tb > 0 && x0 < x1 && x0 >= base && x0 < base + (long long)tb * Hkv) {
      sched[0] = b;
      sched[1] = (int)((x0 - base) / tb);
      sched[2] = (int)((x0 - base) % tb);
    }
    run += tb;
  }
  __syncthreads();
}

// Largest range index r with floor(r * T / R) <= x (the range holding tile x).
__device__ __forceinline__ long long range_of(long long x, long long T, long long R) {
  return ((x + 1) * R + T - 1) / T - 1;
}

// (m, l) <- the log-sum-exp statistics of the union of two sets: maximum m
// and sum of exp(x - m).  Symmetric in its two operands (bit for bit), so
// both lanes of a butterfly exchange end with the same value.
__device__ __forceinline__ void merge_stat(float& m, float& l, float m2, float l2) {
  if (m2 == -INFINITY) return;
  if (m == -INFINITY) {
    m = m2;
    l = l2;
    return;
  }
  const float M = fmaxf(m, m2);
  l = l * __expf(m - M) + l2 * __expf(m2 - M);
  m = M;
}

// Arrival on a unit's counter after this CTA wrote its piece of the unit
// (ntiles of the unit's tb key tiles).  Called by every thread of the
// softmax warps (each warp converged) after its partial-output stores; the
// warps meet on two mbarriers with bounded waits (done: every warp's stores
// issued; flag: the leader warp's verdict), phase `parity`.  One thread
// updates the counter with an acquire-release atomic at GPU scope, whose
// release covers the CTA's stores (they precede it through the `done`
// barrier) and whose acquire, in the CTA that completes the unit, makes
// every other piece visible to the merge that follows.  Returns in every
// caller whether this CTA completed the unit.  The counters were zeroed by
// the kernel before this one in the stream; griddepcontrol.wait waits for it.
__device__ __forceinline__ bool arrive_last(unsigned int* counter, int ntiles, int tb,
                                            uint32_t bar_done, uint32_t bar_flag,
                                            uint32_t parity, bool leader, volatile int* flag,
                                            volatile int* abort, uint64_t timeout_ns) {
  const int lane = threadIdx.x & 31;
  __syncwarp();
  if (lane == 0) mbar_arrive(bar_done);
  if (leader) {
    const bool ok = mbar_wait_warp(bar_done, parity, abort, timeout_ns, 19);
    if (lane == 0) {
      int last = 0;
      if (ok) {
        pdl_wait();
        unsigned int old;
        asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;"
                     : "=r"(old)
                     : "l"(counter), "r"((unsigned int)ntiles)
                     : "memory");
        last = old + (unsigned int)ntiles == (unsigned int)tb;
      }
      *flag = last;
      mbar_arrive(bar_flag);
    }
    __syncwarp();
  }
  return mbar_wait_warp(bar_flag, parity, abort, timeout_ns, 20) && *flag != 0;
}

// Merge of the pieces s = 0 .. n-1 of one unit (workspace slots slot0 + s)
// for columns [c0, c0 + ncol) of the unit's GC and d_v elements [d0, d0 +
// 4 * F4 * TPC) of each: out = sum_s exp(lse_s - L) o_s, L = log sum_s
// exp(lse_s), adding the pieces in range order (bitwise reproducible
// whichever CTA merges).  A group of TPC adjacent lanes per column (TPC a
// power of two <= 32), F4 float4 per thread; t in [0, TPC * ncol) -- other
// threads return.  L: each lane of the group folds every TPC-th piece, then
// a butterfly of symmetric merges gives every lane the same L; the
// weighted sum then takes PP pieces per round with all their loads in
// flight.  With write_lse, L goes to the output LSE.  Loads bypass L1: the
// pieces were written by other SMs.
template <bool BF16, int TPC, int F4>
__device__ __forceinline__ void merge_unit(const DecodeParams& p, int DV, int GC, long long slot0,
                                           int n, int b, int kvh, int c0, int ncol, int d0,
                                           bool write_lse, int t) {
  constexpr int PP = F4 >= 16 ? 1 : 16 / F4;  // pieces per round: <= 16 float4 loads in flight
  const int cc = t / TPC, j = t % TPC;
  if (cc >= ncol) return;  // whole groups leave together
  const int lane = threadIdx.x & 31;
  const unsigned int gmask = (TPC >= 32) ? 0xffffffffu
                                         : (((1u << TPC) - 1u) << (lane & ~(TPC - 1) & 31));
  const int col = c0 + cc;
  const float* lse_c = p.ws_lse + slot0 * GC + col;
  float m = -INFINITY, l = 0.f;
  for (int s = j; s < n; s += TPC) merge_stat(m, l, __ldcg(lse_c + (long long)s * GC), 1.f);
#pragma unroll
  for (int o = TPC / 2; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(gmask, m, o);
    const float l2 = __shfl_xor_sync(gmask, l, o);
    merge_stat(m, l, m2, l2);
  }
  const float L = (m == -INFINITY || !(l > 0.f)) ? -INFINITY : m + __logf(l);
  float4 acc[F4];
#pragma unroll
  for (int k = 0; k < F4; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
  if (L != -INFINITY) {
    const float4* o_c = reinterpret_cast<const float4*>(p.ws_o + (slot0 * GC + col) * (long long)DV + d0);
    const long long piece_f4 = (long long)GC * DV / 4;
    for (int s = 0; s < n; s += PP) {
      float w[PP];
      float4 v[PP][F4];
#pragma unroll
      for (int q = 0; q < PP; ++q) {
        const bool in = s + q < n;
        w[q] = in ? __ldcg(lse_c + (long long)(s + q) * GC) : -INFINITY;
#pragma unroll
        for (int k = 0; k < F4; ++k)
          v[q][k] = in ? __ldcg(o_c + (s + q) * piece_f4 + j + k * TPC) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int q = 0; q < PP; ++q) {  // pieces in range order
        const float wq = s + q < n ? __expf(w[q] - L) : 0.f;
#pragma unroll
        for (int k = 0; k < F4; ++k) {
          acc[k].x = fmaf(wq, v[q][k].x, acc[k].x);
          acc[k].y = fmaf(wq, v[q][k].y, acc[k].y);
          acc[k].z = fmaf(wq, v[q][k].z, acc[k].z);
          acc[k].w = fmaf(wq, v[q][k].w, acc[k].w);
        }
      }
    }
  }
  const int h = kvh * p.G + col / p.Sq, qi = col % p.Sq;
  uint8_t* orow = reinterpret_cast<uint8_t*>(p.out) +
                  ((int64_t)b * p.o_sb + (int64_t)h * p.o_sh + (int64_t)qi * p.o_ss + d0) * 2;
#pragma unroll
  for (int k = 0; k < F4; ++k)
    *reinterpret_cast<uint2*>(orow + (j + k * TPC) * 8) =
        make_uint2(pack2(acc[k].x, acc[k].y, BF16), pack2(acc[k].z, acc[k].w, BF16));
  if (write_lse && j == 0 && p.lse) p.lse[((int64_t)b * p.Hq + h) * p.Sq + qi] = L;
}

// The merge of (b, kv head) pieces, located from one of them: the piece
// starting at global tile gstart, tile0 tiles into its unit of tb tiles.
// Returns the first workspace slot and the number of pieces.
__device__ __forceinline__ int unit_pieces(long long gstart, int tile0, int tb, int unit,
                                           const long long* pos, long long& slot0) {
  const long long su = gstart - tile0;  // the unit's first global tile
  const long long r_lo = range_of(su, pos[1], pos[2]);
  slot0 = r_lo + unit;
  return (int)(range_of(su + tb - 1, pos[1], pos[2]) - r_lo + 1);
}

// Zeroes the arrival counters of the in-kernel merge and writes the output
// of sequences with no key (out = 0, LSE = -inf): no piece covers them.
// Launched with programmatic stream serialization, so that it is resident
// before the previous kernel of the stream ends; it waits for that kernel
// (and all earlier work) to complete, then lets the decode kernel, launched
// after it the same way, start at once -- that kernel reads its inputs
// right away and waits for this one to finish only before its first counter
// update.
template <bool BF16>
__global__ void __launch_bounds__(256) decode_prepare_kernel(const DecodeParams p, int n_counters,
                                                             int DV) {
  pdl_wait();
  pdl_launch_dependents();
  const int tid = blockIdx.x * blockDim.x + threadIdx.x;
  const int nth = gridDim.x * blockDim.x;
  for (int i = tid; i < n_counters; i += nth) p.counters[i] = 0;
  const int rows = p.Hq * p.Sq;
  for (int b = 0; b < p.B; ++b) {
    if (p.skv[b] != 0) continue;
    for (int i = tid; i < rows * (DV / 8); i += nth) {
      const int row = i / (DV / 8), c8 = i % (DV / 8);
      const int h = row / p.Sq, qi = row % p.Sq;
      *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(p.out) +
                                ((int64_t)b * p.o_sb + (int64_t)h * p.o_sh + (int64_t)qi * p.o_ss +
                                 c8 * 8) * 2) = make_uint4(0u, 0u, 0u, 0u);
      if (c8 == 0 && p.lse) p.lse[((int64_t)b * p.Hq + h) * p.Sq + qi] = -INFINITY;
    }
  }
}

template <int DK, int DV, int NH, bool BF16>
__global__ void __launch_bounds__(DecodeTraits<DK, DV, NH>::THREADS, DecodeTraits<DK, DV, NH>::CTAS)
    decode_split_kernel(const __grid_constant__ CUtensorMap tmQ,
                        const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const DecodeParams p) {
  using T = DecodeTraits<DK, DV, NH>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);

  const int hb = blockIdx.x % p.head_blocks;     // head block of the group
  const int rng = blockIdx.x / p.head_blocks;    // key range
  // The N dimension holds "columns" (head g of the group, query i), column
  // g * Sq + i; NH columns per CTA (NH / Sq heads x Sq queries).
  const int GC = p.G * p.Sq;                     // columns per kv head
  const int nvalid = min(NH, GC - hb * NH);      // real columns among the NH rows

  const uint32_t ring = sbase + T::OFF_RING;
  const uint32_t qt = sbase + T::OFF_QT;
  const uint32_t pt = sbase + T::OFF_PT;
  float* red = reinterpret_cast<float*>(smem + T::OFF_RED);
  float* m_sm = reinterpret_cast<float*>(smem + T::OFF_M);
  float* alpha_sm = reinterpret_cast<float*>(smem + T::OFF_ALPHA);
  float* l_sm = reinterpret_cast<float*>(smem + T::OFF_L);
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
  const uint32_t s_full = bar0 + 8u * (2 * T::RING_G);    // [2]
  const uint32_t s_free = s_full + 16;                    // [2]
  const uint32_t p_full = s_free + 16;                    // [NPT]
  const uint32_t o_done = p_full + 8 * T::NPT;            // [NPT]
  const uint32_t q_full = o_done + 8 * T::NPT;           // [NQ]
  const uint32_t q_free = q_full + 8 * T::NQ;             // [NQ]
  const uint32_t red_full = q_free + 8 * T::NQ;           // [2]
  const uint32_t stat_ready = red_full + 16;              // [2]
  const uint32_t drain = stat_ready + 16;
  const uint32_t mg_done = drain + 8;     // in-kernel merge: the softmax warps' stores fenced
  const uint32_t mg_flag = mg_done + 8;   // in-kernel merge: this CTA completed the unit

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int g = 0; g < T::RING_G; ++g) {
      mbar_init(full_bar(g), 1);
      mbar_init(empty_bar(g), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full + 8 * i, 1);
      mbar_init(s_free + 8 * i, T::SOFTMAX_THREADS);
      mbar_init(red_full + 8 * i, T::SOFTMAX_THREADS);
      mbar_init(stat_ready + 8 * i, NH);
    }
    for (int i = 0; i < T::NPT; ++i) {
      mbar_init(p_full + 8 * i, T::SOFTMAX_THREADS);
      mbar_init(o_done + 8 * i, 1);
    }
    for (int i = 0; i < T::NQ; ++i) {
      mbar_init(q_full + 8 * i, 1);
      mbar_init(q_free + 8 * i, 1);
    }
    mbar_init(drain, 1);
    mbar_init(mg_done, T::SOFTMAX_THREADS / 32);
    mbar_init(mg_flag, 1);
    flags[0] = 0;
    flags[1] = 0;
    flags[2] = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), T::TMEM_COLS);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) pdl_launch_dependents();  // the combine may be scheduled now
  locate_range(p.skv, p.B, p.Hkv, 7, p.ranges, rng, scan, sched, pos);  // contains __syncthreads
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int count = sched[3];
  auto walker = [&]() {
    PieceWalker w;
    w.skv = p.skv;
    w.B = p.B;
    w.Hkv = p.Hkv;
    w.shift = 7;
    w.b = sched[0];
    w.kvh = sched[1];
    w.off = sched[2];
    w.remaining = count;
    w.gpos = pos[0];
    return w;
  };

  if (count > 0) {
    if (warp == 0 && lane == 0) {
      // ------------------------------------------------ producer: K/V ring
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      const uint64_t pol = l2_policy_evict_first();
      int grp = 0;
      uint32_t ph = 0;
      bool ok = true;
      // chunks [ch, ch + GCH) of key rows [tok, tok + 128) -> the next ring group
      auto load = [&](const CUtensorMap* map, int ch, int tok, int kvh, int b) {
        if (!ok) return;
        ok = mbar_wait(empty_bar(grp), ph ^ 1u, abort_flag, p.timeout_ns, 1);
        if (!ok) return;
        mbar_arrive_expect_tx(full_bar(grp), T::GBYTES);
        tma_load_5d(ring + grp * T::GBYTES, map, full_bar(grp), 0, tok, ch, kvh, b, pol);
        if (++grp == T::RING_G) { grp = 0; ph ^= 1u; }
      };
      PieceWalker w = walker();
      int b, kvh, t0, n;
      int pv_tok = 0, pv_kvh = 0, pv_b = 0;  // tile whose V is still to be loaded
      bool have_prev = false;
      auto load_v = [&]() {
        for (int c = 0; c < T::VCH; c += T::GCH) load(&tmV, c, pv_tok, pv_kvh, pv_b);
      };
      while (ok && w.next(b, kvh, t0, n)) {
        // A sequence's partial last tile is read as the 128 rows that end at
        // its last key (the rows before the tile are masked): every row read
        // is then a key of the sequence, so whatever the cache holds past
        // skv -- unwritten memory, NaN -- never meets a zero weight in P.V.
        // A sequence shorter than the tile starts at a negative row, which
        // the copy fills with zeros.
        const int last_win = p.skv[b] - T::TILE;
        for (int i = 0; i < n && ok; ++i) {
          const int tok = min((t0 + i) * T::TILE, last_win);
          if (i == 0 && have_prev) load_v();  // finish the previous piece first
          for (int c = 0; c < T::KCH; c += T::GCH) load(&tmK, c, tok, kvh, b);
          if (i > 0) load_v();
          pv_tok = tok;
          pv_kvh = kvh;
          pv_b = b;
          have_prev = true;
        }
      }
      if (have_prev) load_v();
    } else if (warp == 0 && lane == 1) {
      // ------------------------------------------------ producer: Q^T per piece
      tma_prefetch_desc(&tmQ);
      const uint64_t pol = l2_policy_evict_first();
      PieceWalker w = walker();
      int b, kvh, t0, n, k = 0;
      bool ok = true;
      while (ok && w.next(b, kvh, t0, n)) {
        const int qb = k % T::NQ;
        if (k >= T::NQ)  // buffer qb was last read by the S^T MMAs of piece k - NQ
          ok = mbar_wait(q_free + 8 * qb, ((k - T::NQ) / T::NQ) & 1, abort_flag, p.timeout_ns, 3);
        if (!ok) break;
        mbar_arrive_expect_tx(q_full + 8 * qb, T::QT_BYTES);
        // box: 64 columns x Sq queries x NH/Sq heads -> Q^T rows g * Sq + i
        for (int c = 0; c < T::KCH; ++c)
          tma_load_4d(qt + qb * T::QT_BYTES + c * T::QT_CHUNK, &tmQ, q_full + 8 * qb, c * 64, 0,
                      kvh * p.G + hb * (NH / p.Sq), b, pol);
        ++k;
      }
    } else if (warp == 1) {
      // ------------------------------------------------ MMA issuer (whole warp,
      // one elected lane issues; waits are polled by the converged warp)
      constexpr uint32_t idS = umma_idesc(128, NH, BF16, false, false);
      constexpr uint32_t idO = umma_idesc(128, NH, BF16, true, true);
      int grp = 0;
      uint32_t ph = 0;
      bool ok = true;
      auto pv = [&](int t, bool first_of_piece) {
        if (!ok) return;
        const int pb = t % T::NPT;
        ok = mbar_wait_warp(p_full + 8 * pb, (t / T::NPT) & 1, abort_flag, p.timeout_ns, 4);
        if (!ok) return;
        tc_fence_after();
        // B = P^T: MN-major, no swizzle; 8x8 core matrices, 8-head groups 128
        // bytes apart (SBO), 8-key groups NH*16 bytes apart (LBO); 16 keys per
        // K step = 2*NH*16 bytes.
        const uint64_t bd0 = umma_sdesc(pt + pb * T::PT_BYTES, NH * 16, 128, SMEM_NOSWIZZLE);
        for (int i = 0; i < T::DVB; ++i) {
          ok = mbar_wait_warp(full_bar(grp), ph, abort_flag, p.timeout_ns, 5);
          if (!ok) return;
          tc_fence_after();
          if (elect_one()) {
            // A = V^T: MN-major, 128-byte swizzle; the two 64-row halves of
            // the 128-row block are the group's two chunks, one chunk apart
            // (LBO); 8-key groups are 1024 bytes apart (SBO); 16 keys per K
            // step = 2048 bytes.
            const uint64_t ad0 = umma_sdesc(ring + grp * T::GBYTES, T::SLOT, 1024, SMEM_SW128);
            const uint32_t d = tmem + T::TMEM_O + i * NH;
            umma_ss(d, ad0, bd0, idO, first_of_piece ? 0u : 1u);
#pragma unroll
            for (int ks = 1; ks < 8; ++ks)
              umma_ss(d, ad0 + (uint64_t)(ks * (2048 >> 4)), bd0 + (uint64_t)(ks * (2 * NH * 16 >> 4)),
                      idO, 1u);
            umma_commit(empty_bar(grp));
          }
          __syncwarp();
          if (++grp == T::RING_G) { grp = 0; ph ^= 1u; }
        }
        if (elect_one()) umma_commit(o_done + 8 * pb);
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
            ok = ok && mbar_wait_warp(q_full + 8 * (k % T::NQ), (k / T::NQ) & 1, abort_flag, p.timeout_ns, 6);
            if (!ok) break;
            tc_fence_after();
          }
          if (j >= 2) ok = mbar_wait_warp(s_free + 8 * sb, ((j >> 1) - 1) & 1, abort_flag, p.timeout_ns, 7);
          if (!ok) break;
          tc_fence_after();
          // K chunks arrive in ring groups of two (eight MMAs per wait); the
          // zero-filled second chunk of an odd count's last group is skipped.
          const uint32_t qbase = qt + (k % T::NQ) * T::QT_BYTES;
          for (int c = 0; c < T::KCH && ok; c += 2) {
            ok = mbar_wait_warp(full_bar(grp), ph, abort_flag, p.timeout_ns, 8);
            if (!ok) break;
            tc_fence_after();
            if (elect_one()) {
              // A = K tile, B = Q^T: both K-major, 128-byte swizzle, 8-row
              // groups 1024 bytes apart; 16 columns per K step = 32 bytes.
              const uint64_t ad0 = umma_sdesc(ring + grp * T::GBYTES, 16, 1024, SMEM_SW128);
              const uint64_t bd0 = umma_sdesc(qbase + c * T::QT_CHUNK, 16, 1024, SMEM_SW128);
              const uint32_t d = tmem + T::TMEM_S + sb * NH;
              umma_ss(d, ad0, bd0, idS, c > 0 ? 1u : 0u);
#pragma unroll
              for (int ks = 1; ks < 4; ++ks) umma_ss(d, ad0 + 2 * ks, bd0 + 2 * ks, idS, 1u);
              if (c + 1 < T::KCH) {
                const uint64_t ad1 = ad0 + (T::SLOT >> 4);
                const uint64_t bd1 = bd0 + (T::QT_CHUNK >> 4);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) umma_ss(d, ad1 + 2 * ks, bd1 + 2 * ks, idS, 1u);
              }
              umma_commit(empty_bar(grp));
            }
            __syncwarp();
            if (++grp == T::RING_G) { grp = 0; ph ^= 1u; }
          }
          if (!ok) break;
          if (elect_one()) {
            umma_commit(s_full + 8 * sb);
            if (i == n - 1) umma_commit(q_free + 8 * (k % T::NQ));  // this piece's Q^T is free
          }
          __syncwarp();
          if (i > 0) pv(j - 1, prev_first);
          prev_first = (i == 0);
        }
        ++k;
      }
      if (ok && j > 0) pv(j - 1, prev_first);
    } else if (warp >= 2) {
      // ------------------------------------------------ softmax + epilogues
      // Two threads per key row: warps w and w+4 share a TMEM lane quarter,
      // each owning half (HH) of the group's heads for that key.
      // Cross-warp exchanges use mbarriers with bounded waits (red_full: all
      // partial values written; stat_ready: per-head statistics published),
      // so a wait that gives up can never strand the other warps on a
      // barrier.  These threads ignore the abort flag: all of them wait on
      // the same barriers, so they either all see one complete or all time out.
      constexpr int HH = NH / 2;
      const int st = threadIdx.x - 64;       // 0..255
      const int half = st >> 7;              // which half of the heads
      const int h0l = half * HH;             // first head (of the NH) of this thread
      const int wq = warp & 3;               // TMEM lane quarter of this warp
      const int row = wq * 32 + lane;        // key row of S^T / d_v row of O^T blocks
      const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
      volatile int own_abort = 0;
      auto wait = [&](uint32_t bar, uint32_t parity, uint32_t id) {
        return mbar_wait_warp(bar, parity, &own_abort, p.timeout_ns, id);
      };
      if (st < NH) m_sm[st] = -INFINITY;
      named_bar_sync(1, T::SOFTMAX_THREADS);

      PieceWalker w = walker();
      int b, kvh, t0, n, j = 0, r = 0, pc = 0;
      long long gstart;
      bool ok = true;
      while (ok && w.next(b, kvh, t0, n, gstart)) {
        const int skv_b = p.skv[b];
        const int64_t slot_id = (int64_t)rng + (int64_t)b * p.Hkv + kvh;  // workspace slot
        float l[HH];
#pragma unroll
        for (int h = 0; h < HH; ++h) l[h] = 0.f;

        for (int i = 0; i < n && ok; ++i, ++j, ++r) {
          const int sb = j & 1;
          const int rb = r & 1;
          const uint32_t rpar = (r >> 1) & 1;
          ok = wait(s_full + 8 * sb, (j >> 1) & 1, 11);
          if (!ok) break;
          tc_fence_after();
          // Column c holds query qi = c % Sq (Sq a power of two), which sees
          // keys <= skv_b - Sq + qi under the causal mask (bottom-right
          // alignment) and keys < skv_b otherwise; with kq = key - (skv_b - Sq)
          // the causal test is kq <= qi.  The rows of a partial last tile
          // are the 128 keys ending at skv_b; those before the tile's start
          // belong to the previous tile and are masked here.
          const int tile0 = (t0 + i) * T::TILE;
          const int key = min(tile0, skv_b - T::TILE) + row;
          const int kq = key - (skv_b - p.Sq);
          const bool in_seq = key >= tile0;
          const int sq_mask = p.Sq - 1;
          // This thread's HH scores of its key (scaled to log2 units, masked),
          // read from TMEM twice: for the maxima and again for the weights,
          // so that only one HH-wide array is live at a time.
          auto load_s = [&](float (&x)[HH]) {
            tmem_ld<HH>(tmem + lane_base + T::TMEM_S + sb * NH + h0l, x);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < HH; ++e) {
              const bool vis = in_seq && (!p.causal || kq <= ((h0l + e) & sq_mask));
              x[e] = vis ? x[e] * p.scale_log2 : -INFINITY;
            }
          };

          // per-head maximum over the tile's 128 keys
          float* rbuf = red + rb * 4 * NH;
          {
            float v[HH];
            load_s(v);
            transposed_warp_max<HH, HH, 16>(v, lane);
            constexpr int HPL = HH >= 32 ? HH / 32 : 1;
            if (HH >= 32 || (lane & (32 / HH - 1)) == 0) {
#pragma unroll
              for (int e = 0; e < HPL; ++e)
                rbuf[wq * NH + h0l + transposed_head<HH>(lane, e)] = v[e];
            }
          }
          mbar_arrive(red_full + 8 * rb);
          ok = wait(red_full + 8 * rb, rpar, 12);
          if (!ok) break;
          if (st == 0) flags[rb ^ 1] = 0;
          if (st < NH) {
            const float tm =
                fmaxf(fmaxf(rbuf[st], rbuf[NH + st]), fmaxf(rbuf[2 * NH + st], rbuf[3 * NH + st]));
            const float mo = m_sm[st];
            // Keep the stale maximum unless the tile's exceeds it by more than
            // 8 (log2 units): exp2(s - m) then stays <= 256, and the final
            // division by the sum accumulated against the same maximum is exact.
            const bool need = tm > mo + 8.f;
            const float mn = need ? tm : mo;
            alpha_sm[st] = need ? ex2(mo - mn) : 1.f;
            m_sm[st] = mn;
            if (need) flags[rb] = 1;
            mbar_arrive(stat_ready + 8 * rb);
          }
          ok = wait(stat_ready + 8 * rb, rpar, 13);
          if (!ok) break;
          const bool any = flags[rb] != 0;
          // this thread's heads' running max and rescale factors (vector loads)
          float mh[HH], ah[HH];
#pragma unroll
          for (int e = 0; e < HH; e += 4) {
            const float4 m4 = *reinterpret_cast<const float4*>(m_sm + h0l + e);
            const float4 a4 = *reinterpret_cast<const float4*>(alpha_sm + h0l + e);
            mh[e] = m4.x; mh[e + 1] = m4.y; mh[e + 2] = m4.z; mh[e + 3] = m4.w;
            ah[e] = a4.x; ah[e + 1] = a4.y; ah[e + 2] = a4.z; ah[e + 3] = a4.w;
          }

          const int pb = j % T::NPT;
          if (j >= T::NPT) {  // P^T buffer pb was last read by PV(j - NPT)
            ok = wait(o_done + 8 * pb, ((j - T::NPT) / T::NPT) & 1, 14);
            if (!ok) break;
          }
          if (any && i > 0) {  // rescale this thread's O^T columns once PV(j-1) has landed
            ok = wait(o_done + 8 * ((j - 1) % T::NPT), ((j - 1) / T::NPT) & 1, 15);
            if (!ok) break;
            tc_fence_after();
#pragma unroll 1
            for (int d = 0; d < T::DVB; ++d) {
              float o[HH];
              const uint32_t ta = tmem + lane_base + T::TMEM_O + d * NH + h0l;
              tmem_ld<HH>(ta, o);
              tmem_wait_ld();
#pragma unroll
              for (int c = 0; c < HH; ++c) o[c] *= ah[c];
              tmem_st<HH>(ta, o);
            }
            tmem_wait_st();
          }
#pragma unroll
          for (int h = 0; h < HH; ++h) l[h] *= ah[h];

          float sv[HH];
          load_s(sv);
          tc_fence_before();
          mbar_arrive(s_free + 8 * sb);

          // P^T row for this key, this thread's HH heads, as MN-major core matrices.
          const uint32_t prow = pt + pb * T::PT_BYTES + (row >> 3) * (NH * 16) + (row & 7) * 16 +
                                (h0l >> 3) * 128;
#pragma unroll
          for (int g = 0; g < HH / 8; ++g) {
            uint32_t u[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int h = g * 8 + 2 * e;
              const float p0 = sv[h] == -INFINITY ? 0.f : ex2(sv[h] - mh[h]);
              const float p1 = sv[h + 1] == -INFINITY ? 0.f : ex2(sv[h + 1] - mh[h + 1]);
              u[e] = pack2(p0, p1, BF16);
              l[h] += p0;
              l[h + 1] += p1;
            }
            st_shared_v4(prow + g * 128, u[0], u[1], u[2], u[3]);
          }
          fence_proxy_async_smem();
          tc_fence_before();
          mbar_arrive(p_full + 8 * pb);
        }
        if (!ok) break;

        // ---------------------------------------------- epilogue of the piece
        {
          const int t = j - 1;  // last tile of the piece
          ok = wait(o_done + 8 * (t % T::NPT), (t / T::NPT) & 1, 16);
          if (!ok) break;
          tc_fence_after();
          const int rb = r & 1;
          const uint32_t rpar = (r >> 1) & 1;
          float* rbuf = red + rb * 4 * NH;
#pragma unroll
          for (int h = 0; h < HH; ++h) {
            float v = l[h];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == 0) rbuf[wq * NH + h0l + h] = v;
          }
          mbar_arrive(red_full + 8 * rb);
          ok = wait(red_full + 8 * rb, rpar, 17);
          if (!ok) break;
          if (st == 0) flags[rb ^ 1] = 0;
          if (st < NH) {
            const float L = (rbuf[st] + rbuf[NH + st]) + (rbuf[2 * NH + st] + rbuf[3 * NH + st]);
            l_sm[st] = L;
            if (st < nvalid)
              p.ws_lse[slot_id * GC + hb * NH + st] =
                  L > 0.f ? (m_sm[st] + __log2f(L)) * 0.69314718055994531f : -INFINITY;
            m_sm[st] = -INFINITY;  // the next piece starts afresh
            mbar_arrive(stat_ready + 8 * rb);
          }
          ok = wait(stat_ready + 8 * rb, rpar, 18);
          if (!ok) break;
          ++r;
#pragma unroll 1
          for (int d = 0; d < T::DVB; ++d) {
            float o[HH];
            tmem_ld<HH>(tmem + lane_base + T::TMEM_O + d * NH + h0l, o);
            tmem_wait_ld();
            const int dd = d * 128 + row;
#pragma unroll
            for (int c = 0; c < HH; ++c) {
              const int h = h0l + c;
              if (h < nvalid) {
                const float L = l_sm[h];
                p.ws_o[(slot_id * GC + hb * NH + h) * DV + dd] = L > 0.f ? o[c] / L : 0.f;
              }
            }
          }
          tc_fence_before();
          // the CTA that completes the unit's (head block's) key tiles merges
          // the unit's pieces into the output
          if (p.counters) {
            const int unit = b * p.Hkv + kvh;
            const int tb = key_tiles(skv_b, 7);
            const bool last = arrive_last(p.counters + (int64_t)unit * p.head_blocks + hb, n, tb,
                                          mg_done, mg_flag, pc & 1, warp == 2, merge_flag,
                                          &own_abort, p.timeout_ns);
            ++pc;
            if (last) {
              long long slot0;
              const int np = unit_pieces(gstart, t0, tb, unit, pos, slot0);
              constexpr int TPC = T::SOFTMAX_THREADS / NH;  // threads per column
              merge_unit<BF16, TPC, DV / 4 / TPC>(p, DV, GC, slot0, np, b, kvh, hb * NH, nvalid,
                                                  0, true, st);
            }
          }
        }
      }
      if (!ok) *abort_flag = 1;
    }
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

#include "combine_kernel.cuh"
