// cache_append.cuh -- write the new token's cached row(s) before a decode step.
//
// In a decode step the model appends the new token's K/V (MLA: its
// [c_kv | k_pe] row) to the cache and then attends over the whole cache
// ("Full 路线" section 三, past_key_value.update followed by the attention
// call; sections 4.2-4.3 for the latent row).  One block per sequence reads
// the sequence's current length skv[b] once, copies the new rows of all its
// kv heads to position skv[b] in 16-byte pieces, and then advances skv[b];
// a sequence already holding max_skv keys is left untouched and reported
// through bit 1 of the device error word.
#pragma once

#include "sm100.cuh"

namespace attn {

struct AppendParams {
  uint8_t* kc;              // K cache [B, Hkv, max_skv, dk] (byte address)
  uint8_t* vc;              // V cache [B, Hkv, max_skv, dv] (unused when !write_v)
  const uint8_t* kn;        // new K rows [B, Hkv, dk]
  const uint8_t* vn;        // new V rows [B, Hkv, dv]
  int32_t* skv;             // [B] lengths (device, advanced by one)
  int B, Hkv, max_skv, dk, dv, write_v;
  int64_t k_sb, k_sh, k_ss, v_sb, v_sh, v_ss;  // element strides of the caches
  int64_t kn_sb, kn_sh, vn_sb, vn_sh;          // element strides of the new rows
};

__global__ void __launch_bounds__(256) cache_append_kernel(const AppendParams p) {
  const int b = blockIdx.x;
  const int pos = p.skv[b];
  const bool room = pos >= 0 && pos < p.max_skv;
  if (room) {
    const int k16 = p.dk / 8, v16 = p.write_v ? p.dv / 8 : 0;  // 16-byte pieces per row
    const int per_head = k16 + v16;
    for (int i = threadIdx.x; i < p.Hkv * per_head; i += blockDim.x) {
      const int h = i / per_head;
      const int c = i % per_head;
      const uint4* src;
      uint4* dst;
      if (c < k16) {
        src = reinterpret_cast<const uint4*>(p.kn + (b * p.kn_sb + h * p.kn_sh) * 2) + c;
        dst = reinterpret_cast<uint4*>(p.kc + (b * p.k_sb + h * p.k_sh + (int64_t)pos * p.k_ss) * 2) + c;
      } else {
        src = reinterpret_cast<const uint4*>(p.vn + (b * p.vn_sb + h * p.vn_sh) * 2) + (c - k16);
        dst = reinterpret_cast<uint4*>(p.vc + (b * p.v_sb + h * p.v_sh + (int64_t)pos * p.v_ss) * 2) +
              (c - k16);
      }
      *dst = *src;
    }
  } else if (threadIdx.x == 0) {
    atomicOr(&g_attn_error, 2u);
  }
  __syncthreads();  // every thread has read skv[b] before it moves
  if (threadIdx.x == 0 && room) p.skv[b] = pos + 1;
}

}  // namespace attn
