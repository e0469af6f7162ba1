// gather_rows.cuh -- compact caller-selected cache rows for a top-k decode.
//
// Sparse attention in the DSA style ("带你了解Attention" section 5.1: an
// indexer picks the top-k cached entries per query token, attention then
// runs over those only) needs, per sequence, the rows at the selected
// positions.  This copies them into a dense cache of n_sel[b] rows per
// sequence, so that the split-KV decode runs on it unchanged.  HBM-bound
// copy: one block per (sequence, kv head, 128 selected rows), the block's
// positions staged in shared memory, four 16-byte loads in flight per
// thread before their stores.  Positions outside [0, skv[b]) are not read
// (the row is zero-filled) and set bit 2 of the device error word.
#pragma once

#include "sm100.cuh"

namespace attn {

struct GatherParams {
  const uint8_t* src;        // [B, H, >= skv[b], d] (byte address)
  uint8_t* dst;              // [B, H, >= topk, d]
  const int32_t* idx;        // [B, topk] positions into src
  const int32_t* n_sel;      // [B] selected positions per sequence (<= topk)
  const int32_t* skv;        // [B] rows of src per sequence
  int32_t* dst_len;          // [B] written: n_sel[b]
  int B, H, topk, d;
  int64_t s_sb, s_sh, s_ss, d_sb, d_sh, d_ss;  // element strides
  int64_t i_sb;                                // element stride of idx rows
};

constexpr int kGatherRows = 128;  // selected rows per block
constexpr int kGatherUnroll = 4;  // 16-byte loads in flight per thread

__global__ void __launch_bounds__(256) gather_rows_kernel(const GatherParams p) {
  __shared__ int32_t pos_s[kGatherRows];
  const int b = blockIdx.z, h = blockIdx.y;
  const int t0 = blockIdx.x * kGatherRows;
  const int n = max(min(p.n_sel[b], p.topk), 0);
  if (h == 0 && blockIdx.x == 0 && threadIdx.x == 0) p.dst_len[b] = n;
  const int rows = min(n - t0, kGatherRows);
  if (rows <= 0) return;
  const int len = p.skv[b];
  for (int r = threadIdx.x; r < rows; r += blockDim.x) {
    const int pos = p.idx[b * p.i_sb + t0 + r];
    pos_s[r] = (pos >= 0 && pos < len) ? pos : -1;
    if (pos < 0 || pos >= len) atomicOr(&g_attn_error, 4u);
  }
  __syncthreads();
  const int p16 = p.d / 8;  // 16-byte pieces per row
  const int total = rows * p16;
  const uint8_t* src = p.src + (b * p.s_sb + h * p.s_sh) * 2;
  uint8_t* dst = p.dst + (b * p.d_sb + h * p.d_sh + (int64_t)t0 * p.d_ss) * 2;
  for (int base = threadIdx.x; base < total; base += kGatherUnroll * blockDim.x) {
    uint4 v[kGatherUnroll];
#pragma unroll
    for (int u = 0; u < kGatherUnroll; ++u) {
      const int i = base + u * blockDim.x;
      v[u] = make_uint4(0, 0, 0, 0);
      if (i < total) {
        const int pos = pos_s[i / p16];
        if (pos >= 0)  // source rows are read once: stream them past the caches
          v[u] = __ldcs(reinterpret_cast<const uint4*>(src + (int64_t)pos * p.s_ss * 2) + i % p16);
      }
    }
#pragma unroll
    for (int u = 0; u < kGatherUnroll; ++u) {
      const int i = base + u * blockDim.x;
      if (i < total)
        *(reinterpret_cast<uint4*>(dst + (int64_t)(i / p16) * p.d_ss * 2) + i % p16) = v[u];
    }
  }
}

}  // namespace attn
