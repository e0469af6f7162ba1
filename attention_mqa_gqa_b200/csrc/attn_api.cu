// attn_api.cu -- the C ABI declared in include/attn_b200.h: argument
// validation, the launch plan (prefill vs split-KV decode, split sizes),
// TMA tensor maps, and kernel launches on the caller's stream.
//
// Single translation unit: the kernels (and the device error word they
// share) are compiled here.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <atomic>
#include <mutex>

#include "../../include/attn_b200.h"
#include "decode_kernel.cuh"
#include "cache_append.cuh"
#include "gather_rows.cuh"
#include "mla_pair_kernel.cuh"
#include "prefill_kernel.cuh"
#include "prefill_ab_kernel.cuh"

namespace {

constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;  // 2 s per device-side wait
std::atomic<uint64_t> g_wait_timeout_ns{kDefaultTimeoutNs};  // read at each launch

// ------------------------------------------------------------------ driver

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 5-D map over a [B, H, S, D] tensor that splits each row into D/64 chunks
// of 64 columns: dims (innermost first) = {64, S, D/64, H, B} with the chunk
// dimension's stride 128 bytes, box = 64 columns x 128 rows x `kch` chunks,
// 128-byte swizzle.  One copy thus lands `kch` consecutive [128 x 64]
// chunk tiles, each in the layout a per-chunk 2-D box would give, so a
// single TMA instruction moves kch * 16 KB (a copy stream of 16 KB boxes is
// limited per CTA well below HBM bandwidth).  D must be a multiple of 64;
// chunks past D/64 are out of range and zero-filled.
bool make_chunk_map(CUtensorMap* map, const void* base, attn_dtype_t dt, uint64_t D, uint64_t S,
                    uint64_t H, uint64_t B, int64_t ss, int64_t sh, int64_t sb, uint32_t kch,
                    uint32_t rows = 128) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc || D % 64 != 0) return false;
  if (S == 1) ss = (int64_t)D;
  if (H == 1) sh = ss * (int64_t)S;
  if (B == 1) sb = sh * (int64_t)H;
  cuuint64_t dims[5] = {64, S, D / 64, H, B};
  cuuint64_t strides[4] = {(cuuint64_t)ss * 2, 128, (cuuint64_t)sh * 2, (cuuint64_t)sb * 2};
  cuuint32_t box[5] = {64, rows, kch, 1, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = enc(map, dt == ATTN_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                   5, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D map over q [B, Hq, 1, D] seen as rows (head) of D columns: box = 64
// columns x `rows` heads, 128-byte swizzle (the decode kernel's Q^T chunks).
// 4-D map over q [B, Hq, Sq, D]: box = 64 columns x Sq queries x
// `heads` heads, 128-byte swizzle; lands as Q^T rows head * Sq + query (the
// decode kernel's columns).
bool make_q_cols_map(CUtensorMap* map, const void* base, attn_dtype_t dt, uint64_t D, uint64_t Sq,
                     uint64_t H, uint64_t B, int64_t ss, int64_t sh, int64_t sb, uint32_t heads) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  if (Sq == 1) ss = (int64_t)D;
  if (H == 1) sh = ss * (int64_t)Sq;
  if (B == 1) sb = sh * (int64_t)H;
  cuuint64_t dims[4] = {D, Sq, H, B};
  cuuint64_t strides[3] = {(cuuint64_t)ss * 2, (cuuint64_t)sh * 2, (cuuint64_t)sb * 2};
  cuuint32_t box[4] = {64, (cuuint32_t)Sq, heads, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, dt == ATTN_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                   4, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_q_rows_map(CUtensorMap* map, const void* base, attn_dtype_t dt, uint64_t D, uint64_t H,
                     uint64_t B, int64_t sh, int64_t sb, uint32_t rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  if (H == 1) sh = (int64_t)D;
  if (B == 1) sb = sh * (int64_t)H;
  cuuint64_t dims[3] = {D, H, B};
  cuuint64_t strides[2] = {(cuuint64_t)sh * 2, (cuuint64_t)sb * 2};
  cuuint32_t box[3] = {64, rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, dt == ATTN_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                   3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int device_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return 148; }
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    return 148;
  }
  return n;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool strides_ok(const attn_strides_t& s) {
  return s.b >= 0 && s.h >= 0 && s.s >= 0 && s.b % 8 == 0 && s.h % 8 == 0 && s.s % 8 == 0;
}

// Resident decode CTAs per SM (must match DecodeTraits<...>::CTAS).
// Decode CTAs resident per SM: two for d_k = 128, one for 512; for MLA (576)
// one CTA per SM, the SMs working in pairs (each pair one cluster of two CTAs).
int decode_ctas_per_sm(int d_k) { return d_k == 128 ? 2 : 1; }
bool decode_pairs(int d_k) { return d_k == 576; }

bool shape_supported(int Sq, int d_k, int d_v) {
  // prefill: GQA/MHA at 128, MQA at 512, and MLA prefill in its expanded
  // (MHA) form: q_head_dim 192 = 128 + 64 rope columns, v_head_dim 128
  if (Sq > 1)
    return (d_k == 128 && d_v == 128) || (d_k == 512 && d_v == 512) || (d_k == 192 && d_v == 128);
  return (d_k == 128 && d_v == 128) || (d_k == 512 && d_v == 512) || (d_k == 576 && d_v == 512);
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Arrival counters of the in-kernel merge: one per (unit, head block), and
// per CTA of the pair for the MLA kernel (each CTA merges its d rows).
size_t merge_counters(int B, int Hkv, int head_blocks, int d_k) {
  return (size_t)B * Hkv * head_blocks * (d_k == 576 ? 2 : 1);
}

// d = 512 prefill runs on SM pairs that split the two matmuls: one CTA
// computes S and the softmax, the other holds O and runs PV (one work item
// = 128 query rows of one head per pair).
bool prefill_split_matmuls(int d_k) { return d_k == 512; }

// Columns (head x query) per decode CTA for d_k in {128, 512}.
constexpr int kDecodeCols = 16;

// A few queries per sequence against a long cache (extend, speculative
// decoding) run through the split-KV decode kernel with the G heads x Sq
// queries of a kv head as MMA columns: Sq a power of two dividing the
// columns of a CTA.  MLA decode (576) takes Sq == 1 only; longer query
// blocks go to the prefill kernel.
bool decode_path(int Sq, int d_k) {
  if (Sq == 1) return true;
  return (d_k == 128 || d_k == 512) && Sq <= kDecodeCols && (Sq & (Sq - 1)) == 0;
}

attn_status_t plan_impl(int B, int Hq, int Hkv, int Sq, int max_skv, int d_k, int d_v,
                        attn_dtype_t dtype, int num_sms, attn_plan_t* pl) {
  if (!pl) return ATTN_EINVAL;
  std::memset(pl, 0, sizeof(*pl));
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Sq <= 0 || max_skv <= 0 || d_k <= 0 || d_v <= 0)
    return ATTN_EINVAL;
  if (Hq % Hkv != 0) return ATTN_EINVAL;
  if (dtype != ATTN_BF16 && dtype != ATTN_FP16) return ATTN_EINVAL;
  if (!shape_supported(Sq, d_k, d_v)) return ATTN_EUNSUPPORTED;
  if (num_sms <= 0) num_sms = device_sm_count();
  const int G = Hq / Hkv;
  if (!decode_path(Sq, d_k)) {
    pl->path = 0;
    pl->dv_parts = prefill_split_matmuls(d_k) ? 1 : d_v / 128;
    const int64_t n_qt = (Sq + 127) / 128;
    const int64_t items = n_qt * Hq * (int64_t)B * pl->dv_parts;  // persistent CTAs walk these
    if (items > 0x7fffffffLL) return ATTN_EUNSUPPORTED;
    if (prefill_split_matmuls(d_k)) {  // clusters of two CTAs, one item per pair
      const int64_t pairs = num_sms / 2;
      pl->grid_ctas = 2 * (items < pairs ? items : pairs);
    } else {
      pl->grid_ctas = items < num_sms ? items : num_sms;
    }
    pl->workspace_bytes = 0;
    return ATTN_OK;
  }
  pl->path = 1;
  // columns (head x query) per CTA (MLA: heads per CTA pair)
  const int NH = d_k == 576 ? attn::MlaPairTraits::NH : kDecodeCols;
  const int GC = G * Sq;
  pl->heads_per_cta = NH;
  pl->head_blocks = (GC + NH - 1) / NH;
  // One persistent wave: every SM runs decode_ctas_per_sm(d_k) CTAs; the
  // key tiles are cut into equal ranges, one per CTA (MLA: per pair) of
  // each head block.
  const int units_per_range = decode_pairs(d_k) ? 2 : 1;
  int ranges = num_sms * decode_ctas_per_sm(d_k) / units_per_range / pl->head_blocks;
  if (ranges < 1) ranges = 1;
  pl->kv_ranges = ranges;
  pl->partials = (int64_t)ranges + (int64_t)B * Hkv;
  pl->grid_ctas = (int64_t)ranges * pl->head_blocks * units_per_range;
  if (pl->grid_ctas > 0x7fffffffLL || (int64_t)B * Hq * Sq > 0x7fffffffLL)
    return ATTN_EUNSUPPORTED;
  const size_t n = (size_t)pl->partials * GC;
  pl->workspace_bytes = align256(n * d_v * sizeof(float)) + align256(n * sizeof(float)) +
                        align256(merge_counters(B, Hkv, pl->head_blocks, d_k) * sizeof(unsigned int));
  return ATTN_OK;
}

template <typename K>
void set_smem(K kernel, int bytes) {
  // idempotent; cheap enough to repeat per launch
  cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

enum : int { PHASE_PARTIAL = 1, PHASE_COMBINE = 2, PHASE_ALL = 3 };

// attn_fwd's decode: decode_prepare_kernel (counters zeroed, empty
// sequences' output written), then the split kernel with the in-kernel
// merge, launched with programmatic stream serialization so that it starts
// while the small kernel runs (it waits for it only before its first
// counter update).
template <bool BF16>
attn_status_t launch_prepare(const attn::DecodeParams& dp, int n_counters, int d_v,
                             cudaStream_t st) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(4, 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, attn::decode_prepare_kernel<BF16>, dp, n_counters, d_v) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ECUDA;
  }
  return ATTN_OK;
}

// The combine is launched with programmatic stream serialization: its blocks
// may be scheduled while the split kernel finishes and wait (griddepcontrol)
// only before reading the partials, so its launch and prologue overlap the
// split kernel's tail.
template <bool BF16>
attn_status_t launch_combine(const attn::DecodeParams& dp, attn::CombineParams cp,
                             cudaStream_t st) {
  (void)dp;
  // Columns per block: as many as keep a block's outputs within 1024 float4
  // (8 per thread), then halved while the grid would leave SMs idle (down to
  // one float4 per thread).
  const int GC = cp.G * cp.Sq;
  const int D4 = cp.DV / 4;
  const long long units = (long long)cp.B * cp.Hkv;
  int cc = 1;
  while (cc * 2 <= GC && cc * 2 * D4 <= 1024 && cc * 2 <= 32) cc *= 2;
  const long long target = 2LL * device_sm_count();
  while (cc > 1 && cc * D4 > attn::kCombineThreads && units * ((GC + cc - 1) / cc) < target) cc /= 2;
  cp.cols = cc;
  cp.col_chunks = (GC + cc - 1) / cc;
  const int fpt = std::max(1, cc * D4 / attn::kCombineThreads);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)(units * cp.col_chunks), 1, 1);
  cfg.blockDim = dim3(attn::kCombineThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  switch (fpt) {
    case 1: e = cudaLaunchKernelEx(&cfg, attn::combine_kernel<BF16, 1>, cp); break;
    case 2: e = cudaLaunchKernelEx(&cfg, attn::combine_kernel<BF16, 2>, cp); break;
    case 4: e = cudaLaunchKernelEx(&cfg, attn::combine_kernel<BF16, 4>, cp); break;
    default: e = cudaLaunchKernelEx(&cfg, attn::combine_kernel<BF16, 8>, cp); break;
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ECUDA;
  }
  return ATTN_OK;
}

template <int DK, int DV, int NH, bool BF16>
attn_status_t launch_decode(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                            const attn::DecodeParams& dp, const attn::CombineParams& cp,
                            const attn_plan_t& pl, cudaStream_t st, int phases, int n_counters) {
  using Tr = attn::DecodeTraits<DK, DV, NH>;
  static_assert(Tr::CTAS == (DK == 128 ? 2 : 1) && DK != 576, "decode_ctas_per_sm out of sync");
  auto kern = attn::decode_split_kernel<DK, DV, NH, BF16>;
  if (phases == PHASE_ALL) {  // merge in the kernel
    if (launch_prepare<BF16>(dp, n_counters, DV, st) != ATTN_OK) return ATTN_ECUDA;
    set_smem(kern, Tr::SMEM_BYTES);
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)pl.grid_ctas, 1, 1);
    cfg.blockDim = dim3(Tr::THREADS, 1, 1);
    cfg.dynamicSmemBytes = Tr::SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, dp) != cudaSuccess) {
      cudaGetLastError();
      return ATTN_ECUDA;
    }
    return ATTN_OK;
  }
  if (phases & PHASE_PARTIAL) {
    attn::DecodeParams dpp = dp;
    dpp.counters = nullptr;  // partials only; attn_decode_combine merges them
    set_smem(kern, Tr::SMEM_BYTES);
    kern<<<(unsigned)pl.grid_ctas, Tr::THREADS, Tr::SMEM_BYTES, st>>>(mq, mk, mv, dpp);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ECUDA;
  }
  if (phases & PHASE_COMBINE) return launch_combine<BF16>(dp, cp, st);
  return ATTN_OK;
}

template <bool BF16, bool GATHER = false>
attn_status_t launch_mla_pair(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                              const attn::DecodeParams& dp, const attn::CombineParams& cp,
                              const attn_plan_t& pl, cudaStream_t st, int phases, int n_counters) {
  using Tr = attn::MlaPairTraits;
  constexpr int threads = GATHER ? Tr::THREADS_GATHER : Tr::THREADS;
  if (phases & PHASE_PARTIAL) {
    const bool fused = phases == PHASE_ALL;  // merge in the kernel
    if (fused && launch_prepare<BF16>(dp, n_counters, Tr::DV, st) != ATTN_OK) return ATTN_ECUDA;
    attn::DecodeParams dpp = dp;
    if (!fused) dpp.counters = nullptr;
    auto kern = attn::mla_pair_kernel<BF16, GATHER>;
    set_smem(kern, Tr::SMEM_BYTES);
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)pl.grid_ctas, 1, 1);
    cfg.blockDim = dim3(threads, 1, 1);
    cfg.dynamicSmemBytes = Tr::SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = fused ? 2 : 1;
    if (cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, dpp) != cudaSuccess) {
      cudaGetLastError();
      return ATTN_ECUDA;
    }
    if (fused) return ATTN_OK;
  }
  if (phases & PHASE_COMBINE) return launch_combine<BF16>(dp, cp, st);
  return ATTN_OK;
}

template <int DK, int DVH, bool BF16>
attn_status_t launch_prefill(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                             const attn::PrefillParams& pp, const attn_plan_t& pl,
                             cudaStream_t st) {
  using Tr = attn::PrefillTraits<DK, DVH>;
  auto kern = attn::prefill_kernel<DK, DVH, BF16>;
  set_smem(kern, Tr::SMEM_BYTES);
  kern<<<(unsigned)pl.grid_ctas, Tr::THREADS, Tr::SMEM_BYTES, st>>>(mq, mk, mv, pp);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ECUDA;
  return ATTN_OK;
}

// Decode-path parameters of one problem: the workspace carved into partial
// outputs, partial LSEs and merge counters (attn_plan's layout).
void decode_params(const attn_plan_t& pl, int B, int Hq, int Hkv, int Sq, const int32_t* skv, int d_k,
                   int d_v, float scale_log2, int causal, attn_strides_t so, void* out, float* lse,
                   void* workspace, attn::DecodeParams* dp, attn::CombineParams* cp) {
  const int G = Hq / Hkv;
  const size_t n = (size_t)pl.partials * G * Sq;
  *dp = attn::DecodeParams{};
  dp->skv = skv;
  dp->ws_o = reinterpret_cast<float*>(workspace);
  dp->ws_lse = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(workspace) +
                                        align256(n * d_v * sizeof(float)));
  dp->B = B;
  dp->Hq = Hq;
  dp->Hkv = Hkv;
  dp->G = G;
  dp->Sq = Sq;
  dp->causal = causal;
  dp->ranges = pl.kv_ranges;
  dp->head_blocks = pl.head_blocks;
  dp->scale_log2 = scale_log2;
  dp->timeout_ns = g_wait_timeout_ns.load(std::memory_order_relaxed);
  dp->counters = reinterpret_cast<unsigned int*>(reinterpret_cast<uint8_t*>(workspace) +
                                                 align256(n * d_v * sizeof(float)) +
                                                 align256(n * sizeof(float)));
  dp->out = out;
  dp->o_sb = so.b;
  dp->o_sh = so.h;
  dp->o_ss = so.s;
  dp->lse = lse;
  *cp = attn::CombineParams{};
  cp->ws_o = dp->ws_o;
  cp->ws_lse = dp->ws_lse;
  cp->skv = skv;
  cp->out = out;
  cp->o_sb = so.b;
  cp->o_sh = so.h;
  cp->o_ss = so.s;
  cp->lse = lse;
  cp->B = B;
  cp->Hq = Hq;
  cp->Hkv = Hkv;
  cp->G = G;
  cp->Sq = Sq;
  cp->DV = d_v;
  cp->ranges = pl.kv_ranges;
  cp->tile_shift = decode_pairs(d_k) ? attn::MlaPairTraits::TILE_SHIFT : 7;
}

template <bool BF16>
attn_status_t launch_prefill_ab(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                                const attn::PrefillParams& pp, const attn_plan_t& pl,
                                cudaStream_t st) {
  using Tr = attn::PrefillABTraits;
  auto kern = attn::prefill_ab_kernel<BF16>;
  set_smem(kern, Tr::SMEM_BYTES);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)pl.grid_ctas, 1, 1);
  cfg.blockDim = dim3(Tr::THREADS, 1, 1);
  cfg.dynamicSmemBytes = Tr::SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, pp) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ECUDA;
  }
  return ATTN_OK;
}

}  // namespace

extern "C" {

attn_status_t attn_plan(int B, int Hq, int Hkv, int Sq, int max_skv, int d_k, int d_v,
                        attn_dtype_t dtype, int num_sms, attn_plan_t* plan) {
  return plan_impl(B, Hq, Hkv, Sq, max_skv, d_k, d_v, dtype, num_sms, plan);
}

size_t attn_workspace_bytes(int B, int Hq, int Hkv, int Sq, int max_skv, int d_k, int d_v) {
  attn_plan_t pl;
  if (plan_impl(B, Hq, Hkv, Sq, max_skv, d_k, d_v, ATTN_BF16, 0, &pl) != ATTN_OK) return 0;
  return pl.workspace_bytes;
}

}  // extern "C"

namespace {

attn_status_t fwd_impl(const void* q, const void* k, const void* v, void* out, float* lse,
                       int B, int Hq, int Hkv, int Sq, const int32_t* skv_per_seq, int max_skv,
                       int d_k, int d_v, float scale, int causal, attn_dtype_t dtype,
                       attn_strides_t sq, attn_strides_t sk, attn_strides_t sv,
                       attn_strides_t so, void* workspace, size_t workspace_bytes,
                       void* cuda_stream, int phases) {
  // ---- validation (nothing touches the GPU before this passes)
  if (!q || !k || !v || !out || !skv_per_seq) return ATTN_EINVAL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return ATTN_EINVAL;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return ATTN_EINVAL;
  if (reinterpret_cast<uintptr_t>(skv_per_seq) & 3u) return ATTN_EINVAL;
  if (!strides_ok(sq) || !strides_ok(sk) || !strides_ok(sv) || !strides_ok(so)) return ATTN_EINVAL;
  if (causal != 0 && causal != 1) return ATTN_EINVAL;
  if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_EINVAL;
  attn_plan_t pl;
  attn_status_t rc = plan_impl(B, Hq, Hkv, Sq, max_skv, d_k, d_v, dtype, 0, &pl);
  if (rc != ATTN_OK) return rc;
  if (phases != PHASE_ALL && pl.path != 1) return ATTN_EINVAL;  // phases exist for decode only
  if ((Sq > 1 && sq.s == 0) || sk.s == 0 || sv.s == 0 || (Sq > 1 && so.s == 0)) return ATTN_EINVAL;
  if (pl.workspace_bytes > 0) {
    if (!workspace || !aligned16(workspace)) return ATTN_EWORKSPACE;
    if (workspace_bytes < pl.workspace_bytes) return ATTN_EWORKSPACE;
  }

  cudaStream_t st = reinterpret_cast<cudaStream_t>(cuda_stream);
  const float scale_log2 = scale * 1.4426950408889634f;
  const bool bf16 = dtype == ATTN_BF16;
  const int G = Hq / Hkv;

  CUtensorMap mk, mv;
  if (pl.path == 1) {
    if ((Hq > 1 && sq.h == 0) || (B > 1 && sq.b == 0)) return ATTN_EINVAL;
    if (!make_chunk_map(&mk, k, dtype, d_k, max_skv, Hkv, B, sk.s, sk.h, sk.b, 2)) return ATTN_ECUDA;
    if (!make_chunk_map(&mv, v, dtype, d_v, max_skv, Hkv, B, sv.s, sv.h, sv.b, 2)) return ATTN_ECUDA;
    CUtensorMap mq;
    if (decode_pairs(d_k)) {
      if (!make_q_rows_map(&mq, q, dtype, d_k, Hq, B, sq.h, sq.b, attn::MlaPairTraits::NHC))
        return ATTN_ECUDA;
    } else if (!make_q_cols_map(&mq, q, dtype, d_k, Sq, Hq, B, sq.s, sq.h, sq.b,
                                (uint32_t)(kDecodeCols / Sq))) {
      return ATTN_ECUDA;
    }
    attn::DecodeParams dp{};
    attn::CombineParams cp{};
    decode_params(pl, B, Hq, Hkv, Sq, skv_per_seq, d_k, d_v, scale_log2, causal, so, out, lse,
                  workspace, &dp, &cp);
    const int n_counters = (int)merge_counters(B, Hkv, pl.head_blocks, d_k);
    if (d_k == 128)
      return bf16 ? launch_decode<128, 128, 16, true>(mq, mk, mv, dp, cp, pl, st, phases, n_counters)
                  : launch_decode<128, 128, 16, false>(mq, mk, mv, dp, cp, pl, st, phases, n_counters);
    if (d_k == 512)
      return bf16 ? launch_decode<512, 512, 16, true>(mq, mk, mv, dp, cp, pl, st, phases, n_counters)
                  : launch_decode<512, 512, 16, false>(mq, mk, mv, dp, cp, pl, st, phases, n_counters);
    return bf16 ? launch_mla_pair<true>(mq, mk, mv, dp, cp, pl, st, phases, n_counters)
                : launch_mla_pair<false>(mq, mk, mv, dp, cp, pl, st, phases, n_counters);
  }

  const bool split = prefill_split_matmuls(d_k);
  // split matmuls: Q and K copies of 4 chunks x 128 rows, V copies of 8
  // chunks x 64 keys (64 KB each); otherwise 2 chunks x 128 rows
  if (!make_chunk_map(&mk, k, dtype, d_k, max_skv, Hkv, B, sk.s, sk.h, sk.b, split ? 4 : 2))
    return ATTN_ECUDA;
  if (!make_chunk_map(&mv, v, dtype, d_v, max_skv, Hkv, B, sv.s, sv.h, sv.b, split ? 8 : 2,
                      split ? 64 : 128))
    return ATTN_ECUDA;
  CUtensorMap mq;
  if (!make_chunk_map(&mq, q, dtype, d_k, Sq, Hq, B, sq.s, sq.h, sq.b, split ? 4 : 2))
    return ATTN_ECUDA;
  attn::PrefillParams pp{};
  pp.out = out;
  pp.o_sb = so.b;
  pp.o_sh = so.h;
  pp.o_ss = so.s;
  pp.lse = lse;
  pp.skv = skv_per_seq;
  pp.B = B;
  pp.Hq = Hq;
  pp.Hkv = Hkv;
  pp.G = G;
  pp.Sq = Sq;
  pp.n_qtiles = (Sq + 127) / 128;
  pp.dv_parts = pl.dv_parts;
  pp.n_items = pp.n_qtiles * Hq * B * pl.dv_parts;  // per CTA, or per pair (split matmuls)
  {
    // K/V bytes of one kv head over the batch; blocks of kv heads whose
    // K/V stays within ~40 MB of the 126 MB L2
    const double kv_head_bytes = (double)B * max_skv * (d_k + d_v) * 2.0;
    int kv_heads = (int)(40.0e6 / (kv_head_bytes > 1.0 ? kv_head_bytes : 1.0));
    if (kv_heads < 1) kv_heads = 1;
    if (kv_heads > Hkv) kv_heads = Hkv;
    pp.heads_per_block = kv_heads * G;
  }
  pp.scale_log2 = scale_log2;
  pp.causal = causal;
  pp.timeout_ns = g_wait_timeout_ns.load(std::memory_order_relaxed);
  if (d_k == 128)
    return bf16 ? launch_prefill<128, 128, true>(mq, mk, mv, pp, pl, st)
                : launch_prefill<128, 128, false>(mq, mk, mv, pp, pl, st);
  if (d_k == 192)
    return bf16 ? launch_prefill<192, 128, true>(mq, mk, mv, pp, pl, st)
                : launch_prefill<192, 128, false>(mq, mk, mv, pp, pl, st);
  return bf16 ? launch_prefill_ab<true>(mq, mk, mv, pp, pl, st)
              : launch_prefill_ab<false>(mq, mk, mv, pp, pl, st);
}

}  // namespace

extern "C" {

#define ATTN_FWD_ARGS                                                                           \
  q, k, v, out, lse, B, Hq, Hkv, Sq, skv_per_seq, max_skv, d_k, d_v, scale, causal, dtype, sq, \
      sk, sv, so, workspace, workspace_bytes, cuda_stream

attn_status_t attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse,
                       int B, int Hq, int Hkv, int Sq, const int32_t* skv_per_seq, int max_skv,
                       int d_k, int d_v, float scale, int causal, attn_dtype_t dtype,
                       attn_strides_t sq, attn_strides_t sk, attn_strides_t sv,
                       attn_strides_t so, void* workspace, size_t workspace_bytes,
                       void* cuda_stream) {
  return fwd_impl(ATTN_FWD_ARGS, PHASE_ALL);
}

attn_status_t attn_decode_partial(const void* q, const void* k, const void* v, void* out,
                                  float* lse, int B, int Hq, int Hkv, int Sq,
                                  const int32_t* skv_per_seq, int max_skv, int d_k, int d_v,
                                  float scale, int causal, attn_dtype_t dtype, attn_strides_t sq,
                                  attn_strides_t sk, attn_strides_t sv, attn_strides_t so,
                                  void* workspace, size_t workspace_bytes, void* cuda_stream) {
  return fwd_impl(ATTN_FWD_ARGS, PHASE_PARTIAL);
}

attn_status_t attn_decode_combine(const void* q, const void* k, const void* v, void* out,
                                  float* lse, int B, int Hq, int Hkv, int Sq,
                                  const int32_t* skv_per_seq, int max_skv, int d_k, int d_v,
                                  float scale, int causal, attn_dtype_t dtype, attn_strides_t sq,
                                  attn_strides_t sk, attn_strides_t sv, attn_strides_t so,
                                  void* workspace, size_t workspace_bytes, void* cuda_stream) {
  return fwd_impl(ATTN_FWD_ARGS, PHASE_COMBINE);
}

attn_status_t attn_last_device_error(void* cuda_stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(cuda_stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return ATTN_ECUDA;
  unsigned int word = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&word, attn::g_attn_error, sizeof(word)) != cudaSuccess)
    return ATTN_ECUDA;
  if (word != 0 && cudaMemcpyToSymbol(attn::g_attn_error, &zero, sizeof(zero)) != cudaSuccess)
    return ATTN_ECUDA;
  if (word & 1u) return ATTN_ETIMEOUT;
  if (word & 2u) return ATTN_EOVERFLOW;
  return word ? ATTN_EINDEX : ATTN_OK;
}

const char* attn_status_str(attn_status_t s) {
  switch (s) {
    case ATTN_OK: return "ok";
    case ATTN_EINVAL: return "invalid argument";
    case ATTN_EUNSUPPORTED: return "unsupported shape or type";
    case ATTN_EWORKSPACE: return "workspace missing or too small";
    case ATTN_ECUDA: return "CUDA error";
    case ATTN_ETIMEOUT: return "device-side wait timed out";
    case ATTN_EOVERFLOW: return "cache full: a sequence already holds max_skv keys";
    case ATTN_EINDEX: return "a selected position lies outside its sequence";
  }
  return "unknown status";
}

const char* attn_version(void) { return "0.1.0"; }

attn_status_t attn_cache_append(void* k_cache, void* v_cache, const void* k_new, const void* v_new,
                                int32_t* skv_per_seq, int B, int Hkv, int max_skv, int d_k,
                                int d_v, attn_dtype_t dtype, attn_strides_t sk, attn_strides_t sv,
                                attn_strides_t skn, attn_strides_t svn, void* cuda_stream) {
  if (!k_cache || !k_new || !skv_per_seq) return ATTN_EINVAL;
  if (B <= 0 || Hkv <= 0 || max_skv <= 0 || d_k <= 0 || d_v < 0) return ATTN_EINVAL;
  if (dtype != ATTN_BF16 && dtype != ATTN_FP16) return ATTN_EINVAL;
  if (d_k % 8 != 0 || d_v % 8 != 0) return ATTN_EINVAL;
  if (reinterpret_cast<uintptr_t>(skv_per_seq) & 3u) return ATTN_EINVAL;
  // v_cache == NULL or == k_cache with d_v <= d_k: the MLA latent cache,
  // where V is a view of K's rows -- only the K row is written
  const bool write_v = v_cache && v_cache != k_cache && d_v > 0;
  if (write_v && !v_new) return ATTN_EINVAL;
  if (!aligned16(k_cache) || !aligned16(k_new) || (write_v && (!aligned16(v_cache) || !aligned16(v_new))))
    return ATTN_EINVAL;
  if (!strides_ok(sk) || !strides_ok(skn) || (write_v && (!strides_ok(sv) || !strides_ok(svn))))
    return ATTN_EINVAL;
  attn::AppendParams ap{};
  ap.kc = reinterpret_cast<uint8_t*>(k_cache);
  ap.vc = reinterpret_cast<uint8_t*>(v_cache);
  ap.kn = reinterpret_cast<const uint8_t*>(k_new);
  ap.vn = reinterpret_cast<const uint8_t*>(v_new);
  ap.skv = skv_per_seq;
  ap.B = B;
  ap.Hkv = Hkv;
  ap.max_skv = max_skv;
  ap.dk = d_k;
  ap.dv = d_v;
  ap.write_v = write_v ? 1 : 0;
  ap.k_sb = sk.b;
  ap.k_sh = sk.h;
  ap.k_ss = sk.s;
  ap.v_sb = sv.b;
  ap.v_sh = sv.h;
  ap.v_ss = sv.s;
  ap.kn_sb = skn.b;
  ap.kn_sh = skn.h;
  ap.vn_sb = svn.b;
  ap.vn_sh = svn.h;
  attn::cache_append_kernel<<<B, 256, 0, reinterpret_cast<cudaStream_t>(cuda_stream)>>>(ap);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ECUDA;
}

attn_status_t attn_topk_fwd(const void* q, const void* cache, void* out, float* lse, int B, int Hq,
                            const int32_t* idx, int64_t idx_stride, const int32_t* n_sel,
                            const int32_t* skv_per_seq, int topk, int max_skv, int d_k, int d_v,
                            float scale, attn_dtype_t dtype, attn_strides_t sq, attn_strides_t sc,
                            attn_strides_t so, void* workspace, size_t workspace_bytes,
                            void* cuda_stream) {
  // ---- validation (nothing touches the GPU before this passes)
  if (!q || !cache || !out || !idx || !n_sel || !skv_per_seq) return ATTN_EINVAL;
  if (d_k != 576 || d_v != 512) return ATTN_EUNSUPPORTED;  // the absorbed-MLA latent cache
  if (B <= 0 || Hq <= 0 || topk <= 0 || max_skv <= 0 || idx_stride < topk) return ATTN_EINVAL;
  if (!aligned16(q) || !aligned16(cache) || !aligned16(out)) return ATTN_EINVAL;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return ATTN_EINVAL;
  for (const void* ptr : {static_cast<const void*>(idx), static_cast<const void*>(n_sel),
                          static_cast<const void*>(skv_per_seq)})
    if (reinterpret_cast<uintptr_t>(ptr) & 3u) return ATTN_EINVAL;
  if (!strides_ok(sq) || !strides_ok(sc) || !strides_ok(so) || sc.s == 0) return ATTN_EINVAL;
  if ((Hq > 1 && sq.h == 0) || (B > 1 && (sq.b == 0 || sc.b == 0))) return ATTN_EINVAL;
  if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_EINVAL;
  attn_plan_t pl;
  attn_status_t rc = plan_impl(B, Hq, 1, 1, topk, d_k, d_v, dtype, 0, &pl);
  if (rc != ATTN_OK) return rc;
  if (pl.workspace_bytes > 0) {
    if (!workspace || !aligned16(workspace)) return ATTN_EWORKSPACE;
    if (workspace_bytes < pl.workspace_bytes) return ATTN_EWORKSPACE;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(cuda_stream);
  CUtensorMap mq, mk, mv;  // K and V come by the kernel's own gathers; the maps stay unused
  if (!make_q_rows_map(&mq, q, dtype, d_k, Hq, B, sq.h, sq.b, attn::MlaPairTraits::NHC))
    return ATTN_ECUDA;
  if (!make_chunk_map(&mk, cache, dtype, d_k, max_skv, 1, B, sc.s, sc.h, sc.b, 2)) return ATTN_ECUDA;
  if (!make_chunk_map(&mv, cache, dtype, d_v, max_skv, 1, B, sc.s, sc.h, sc.b, 2)) return ATTN_ECUDA;
  attn::DecodeParams dp{};
  attn::CombineParams cp{};
  decode_params(pl, B, Hq, 1, 1, n_sel, d_k, d_v, scale * 1.4426950408889634f, 0, so, out, lse,
                workspace, &dp, &cp);
  dp.idx = idx;
  dp.idx_sb = idx_stride;
  dp.src = reinterpret_cast<const uint8_t*>(cache);
  dp.src_sb = sc.b;
  dp.src_ss = sc.s;
  dp.src_len = skv_per_seq;
  const int n_counters = (int)merge_counters(B, 1, pl.head_blocks, d_k);
  return dtype == ATTN_BF16
             ? launch_mla_pair<true, true>(mq, mk, mv, dp, cp, pl, st, PHASE_ALL, n_counters)
             : launch_mla_pair<false, true>(mq, mk, mv, dp, cp, pl, st, PHASE_ALL, n_counters);
}

attn_status_t attn_gather_rows(const void* src, void* dst, const int32_t* idx,
                               const int32_t* n_sel, const int32_t* skv_per_seq, int32_t* dst_len,
                               int B, int H, int topk, int d, attn_dtype_t dtype,
                               attn_strides_t s_src, attn_strides_t s_dst, int64_t idx_stride,
                               void* cuda_stream) {
  if (!src || !dst || !idx || !n_sel || !skv_per_seq || !dst_len) return ATTN_EINVAL;
  if (B <= 0 || H <= 0 || topk <= 0 || d <= 0 || d % 8 != 0 || idx_stride < topk) return ATTN_EINVAL;
  if (dtype != ATTN_BF16 && dtype != ATTN_FP16) return ATTN_EINVAL;
  if (!aligned16(src) || !aligned16(dst) || !strides_ok(s_src) || !strides_ok(s_dst))
    return ATTN_EINVAL;
  for (const void* q : {static_cast<const void*>(idx), static_cast<const void*>(n_sel),
                        static_cast<const void*>(skv_per_seq), static_cast<const void*>(dst_len)})
    if (reinterpret_cast<uintptr_t>(q) & 3u) return ATTN_EINVAL;
  if (B > 65535 || H > 65535) return ATTN_EUNSUPPORTED;
  attn::GatherParams gp{};
  gp.src = reinterpret_cast<const uint8_t*>(src);
  gp.dst = reinterpret_cast<uint8_t*>(dst);
  gp.idx = idx;
  gp.n_sel = n_sel;
  gp.skv = skv_per_seq;
  gp.dst_len = dst_len;
  gp.B = B;
  gp.H = H;
  gp.topk = topk;
  gp.d = d;
  gp.s_sb = s_src.b;
  gp.s_sh = s_src.h;
  gp.s_ss = s_src.s;
  gp.d_sb = s_dst.b;
  gp.d_sh = s_dst.h;
  gp.d_ss = s_dst.s;
  gp.i_sb = idx_stride;
  const dim3 grid((unsigned)((topk + 127) / 128), (unsigned)H, (unsigned)B);
  attn::gather_rows_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(cuda_stream)>>>(gp);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ECUDA;
}

uint64_t attn_set_wait_timeout_ns(uint64_t ns) {
  return g_wait_timeout_ns.exchange(ns == 0 ? kDefaultTimeoutNs : ns);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// attn_fwd_noalloc: attn_fwd for callers that cannot allocate device memory.
//
// The decode path needs scratch memory (per-split partial outputs and LSEs)
// that attn_fwd takes from a caller-provided workspace.  Some callers cannot
// obtain one: a plugin run by a host framework that owns all device memory
// and hands plugins no allocator, or a latency-critical loop where
// cudaMalloc's implicit device-wide synchronisation is not acceptable.  This
// entry point uses a fixed buffer compiled into the library instead.
//
// The buffer is a file-scope __device__ array of ATTN_NOALLOC_SCRATCH_BYTES;
// every GPU that loads the library holds it until the process exits.  Host
// code cannot pass the array's name to a kernel (on the host it only names a
// stand-in object), so its device address is looked up once per device with
// cudaGetSymbolAddress, with that device current, on the first call made on
// that device (and looked up again if the device's context has been
// replaced since, e.g. after cudaDeviceReset).  All calls share the buffer
// and it keeps whatever the last call left there; the kernels write every
// scratch value before reading it, so nothing has to be cleared between
// calls.  Calls that overlap on the GPU (other streams, other host threads)
// race on the buffer.
// ---------------------------------------------------------------------------

namespace {

static __device__ __align__(256) uint8_t g_noalloc_scratch[ATTN_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};
CUcontext g_noalloc_ctx[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

// The calling thread's current CUDA context (null if it cannot be told).
CUcontext current_context() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  CUcontext c = nullptr;
  if (!fn || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

// Device address of g_noalloc_scratch on the current device: looked up on
// the first call on the device and again whenever the device's context is
// not the one the cached address was taken in.
attn_status_t noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return ATTN_ECUDA; }
  if (dev < 0 || dev >= kMaxDevices) return ATTN_EUNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  CUcontext ctx = current_context();
  if (!g_noalloc_ptr[dev] || !ctx || ctx != g_noalloc_ctx[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return ATTN_ECUDA;
    }
    g_noalloc_ptr[dev] = p;
    // the lookup makes the device's primary context current if none was
    g_noalloc_ctx[dev] = ctx ? ctx : current_context();
  }
  *out = g_noalloc_ptr[dev];
  return ATTN_OK;
}

}  // namespace

extern "C" attn_status_t attn_fwd_noalloc(const void* q, const void* k, const void* v, void* out,
                                          float* lse, int B, int Hq, int Hkv, int Sq,
                                          const int32_t* skv_per_seq, int max_skv, int d_k,
                                          int d_v, float scale, int causal, attn_dtype_t dtype,
                                          attn_strides_t sq, attn_strides_t sk,
                                          attn_strides_t sv, attn_strides_t so,
                                          void* cuda_stream) {
  // Size check first: a problem whose scratch would not fit is refused
  // before anything touches the device.
  attn_plan_t pl;
  attn_status_t rc = plan_impl(B, Hq, Hkv, Sq, max_skv, d_k, d_v, dtype, 0, &pl);
  if (rc != ATTN_OK) return rc;
  if (pl.workspace_bytes > (size_t)ATTN_NOALLOC_SCRATCH_BYTES) return ATTN_EWORKSPACE;
  void* scratch = nullptr;
  if (pl.workspace_bytes > 0) {
    rc = noalloc_scratch(&scratch);
    if (rc != ATTN_OK) return rc;
  }
  return fwd_impl(q, k, v, out, lse, B, Hq, Hkv, Sq, skv_per_seq, max_skv, d_k, d_v, scale,
                  causal, dtype, sq, sk, sv, so, scratch, (size_t)ATTN_NOALLOC_SCRATCH_BYTES,
                  cuda_stream, PHASE_ALL);
}
