// combine_kernel.cuh -- merge the split-KV decode partials of each query row.
//
// out[b,h,i,:] = sum_s exp(lse_s - L) o_s,  L = log sum_s exp(lse_s), over
// the pieces s of unit (b, h / G), in range order (no atomics, so the result
// is bitwise reproducible: "GQA和MLA详解" section 4 on reduction order).  The
// pieces are the normalised partial outputs o_s and log-sum-exps lse_s the
// partial kernels write per (key range, unit); this is the merge of softmax
// results over disjoint key subsets.
#pragma once

#include "decode_kernel.cuh"

namespace attn {

struct CombineParams {
  const float* ws_o;
  const float* ws_lse;
  const int32_t* skv;
  void* out;
  int64_t o_sb, o_sh;
  int64_t o_ss;
  float* lse;  // [B, Hq, Sq] or NULL
  int B, Hq, Hkv, G, DV, ranges;
  int Sq;          // queries per sequence (columns per head)
  int tile_shift;  // log2 of the keys per tile the partial kernel used
  int cols;        // columns (of the unit's G * Sq) per block: a power of two <= 32
  int col_chunks;  // blocks per unit = ceil(G * Sq / cols)
};

constexpr int kCombineThreads = 128;

// One block per (unit u = (b, kv head), chunk of `cols` columns).  The
// pieces of a unit are the same for all its G * Sq columns, and piece s of
// every column lives in workspace slot (r_lo + s) + u, where the columns'
// partial rows are contiguous: the block finds the unit's pieces once, then
//  1. each column's L: a group of `per` adjacent lanes per column, each lane
//     folding every per-th piece, merged by a butterfly over the group; when
//     all pieces fit one pass (n <= per) each lane turns the one lse it read
//     into its weight exp(lse - L) in shared memory right away;
//  2. otherwise the weights of up to W pieces at a time are staged;
//  3. the weighted sum: thread t owns FPT float4 positions of the block's
//     cols x d_v outputs and keeps 16 loads in flight (16 / FPT pieces per
//     round), adding the pieces in range order.
template <bool BF16, int FPT>
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(const CombineParams p) {
  constexpr int NT = kCombineThreads;
  constexpr int W = 2048;      // staged weights (pieces x columns)
  constexpr int LIF = 16;      // float4 loads in flight per thread
  constexpr int PPI = LIF / FPT;
  __shared__ float w_sm[W];
  __shared__ float L_sm[32];
  __shared__ long long redl[8];
  const int CC = p.cols;
  const int chunk = blockIdx.x % p.col_chunks;
  const int unit = blockIdx.x / p.col_chunks;
  const int b = unit / p.Hkv, kvh = unit % p.Hkv;
  const int GC = p.G * p.Sq;
  const int c0 = chunk * CC;
  const int ncol = min(CC, GC - c0);
  const int t = threadIdx.x;
  const int warp = t >> 5, lane = t & 31;

  // tiles of the sequences before b, and of all sequences
  long long pre = 0, tot = 0;
  for (int bb = t; bb < p.B; bb += NT) {
    const int tb = key_tiles(p.skv[bb], p.tile_shift);
    tot += tb;
    if (bb < b) pre += tb;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    pre += __shfl_xor_sync(0xffffffffu, pre, o);
    tot += __shfl_xor_sync(0xffffffffu, tot, o);
  }
  if (lane == 0) {
    redl[warp] = pre;
    redl[4 + warp] = tot;
  }
  __syncthreads();
  pre = (redl[0] + redl[1]) + (redl[2] + redl[3]);
  tot = (redl[4] + redl[5]) + (redl[6] + redl[7]);
  const int tu = key_tiles(p.skv[b], p.tile_shift);
  const long long T = tot * p.Hkv;
  // Everything above reads inputs only; the partials come from the kernel
  // before this one in the stream, which may still be running.
  pdl_wait();
  const long long Re = T < p.ranges ? T : p.ranges;  // ranges in use, none empty
  int n = 0;
  long long r_lo = 0;
  if (tu > 0) {
    const long long su = pre * p.Hkv + (long long)kvh * tu;
    r_lo = range_of(su, T, Re);
    n = (int)(range_of(su + tu - 1, T, Re) - r_lo + 1);
  }
  const long long slot0 = r_lo + unit;  // piece s: slot slot0 + s
  const float* lse_base = p.ws_lse + slot0 * GC + c0;

  // 1. per-column statistics (all lanes take part in the shuffles)
  const int per = min(32, NT / CC);  // lanes per column, a power of two
  const int c = t / per, j = t % per;
  float m = -INFINITY, l = 0.f, x0 = -INFINITY;
  if (c < ncol) {
    for (int s = j; s < n; s += per) {
      const float x = lse_base[(long long)s * GC + c];
      if (s == j) x0 = x;
      merge_stat(m, l, x, 1.f);
    }
  }
  for (int o = per >> 1; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float l2 = __shfl_xor_sync(0xffffffffu, l, o);
    merge_stat(m, l, m2, l2);
  }
  const float L = (m == -INFINITY || !(l > 0.f)) ? -INFINITY : m + __logf(l);
  if (j == 0 && c < ncol) L_sm[c] = L;
  const bool one_pass = n <= per;  // then n * CC <= 32 * 32 <= W
  if (one_pass && c < ncol && j < n) w_sm[j * CC + c] = L == -INFINITY ? 0.f : __expf(x0 - L);
  __syncthreads();

  // 2-3. weighted sum of the pieces
  const int D4 = p.DV >> 2;  // float4 per column
  const int nf = ncol * D4;  // float4 outputs of this block
  const float4* o_base = reinterpret_cast<const float4*>(p.ws_o + (slot0 * GC + c0) * (long long)p.DV);
  const long long piece_f4 = (long long)GC * D4;
  float4 acc[FPT];
#pragma unroll
  for (int k = 0; k < FPT; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
  const int PB = W / CC;  // pieces per weight batch (>= 64)
  for (int sb = 0; sb < n; sb += PB) {
    const int nb = min(PB, n - sb);
    if (!one_pass) {
      for (int i = t; i < nb * CC; i += NT) {
        const int cc = i % CC;
        const float Lc = cc < ncol ? L_sm[cc] : -INFINITY;
        w_sm[i] = Lc == -INFINITY ? 0.f
                                  : __expf(lse_base[(long long)(sb + i / CC) * GC + cc] - Lc);
      }
      __syncthreads();
    }
    for (int s = 0; s < nb; s += PPI) {
      float4 v[LIF];
#pragma unroll
      for (int i = 0; i < LIF; ++i) {
        const int k = i % FPT, so = i / FPT;
        const int f = t + NT * k;
        v[i] = (s + so < nb && f < nf) ? o_base[(long long)(sb + s + so) * piece_f4 + f]
                                       : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int i = 0; i < LIF; ++i) {  // for each k, pieces in increasing order
        const int k = i % FPT, so = i / FPT;
        const int f = t + NT * k;
        if (s + so < nb && f < nf) {
          const float wv = w_sm[(s + so) * CC + f / D4];
          acc[k].x = fmaf(wv, v[i].x, acc[k].x);
          acc[k].y = fmaf(wv, v[i].y, acc[k].y);
          acc[k].z = fmaf(wv, v[i].z, acc[k].z);
          acc[k].w = fmaf(wv, v[i].w, acc[k].w);
        }
      }
    }
    if (!one_pass) __syncthreads();
  }
#pragma unroll
  for (int k = 0; k < FPT; ++k) {
    const int f = t + NT * k;
    if (f < nf) {
      const int col = c0 + f / D4;
      const int h = kvh * p.G + col / p.Sq, qi = col % p.Sq;
      uint8_t* outp = reinterpret_cast<uint8_t*>(p.out) +
                      ((int64_t)b * p.o_sb + (int64_t)h * p.o_sh + (int64_t)qi * p.o_ss +
                       (f % D4) * 4) * 2;
      *reinterpret_cast<uint2*>(outp) =
          make_uint2(pack2(acc[k].x, acc[k].y, BF16), pack2(acc[k].z, acc[k].w, BF16));
    }
  }
  if (t < ncol && p.lse) {
    const int col = c0 + t;
    const int h = kvh * p.G + col / p.Sq, qi = col % p.Sq;
    p.lse[((int64_t)b * p.Hq + h) * p.Sq + qi] = L_sm[t];
  }
}

}  // namespace attn
