// attn_api.cu - the C ABI declared in include/attn.h: host-side argument
// checks, TMA tensor-map encoding, work decomposition and kernel launches.
// Nothing here allocates device memory or synchronises a stream.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/attn.h"
#include "aux_kernels.cuh"
#include "bwd_kernel.cuh"
#include "fwd_kernel.cuh"
#include "kvcache_kernel.cuh"

using namespace attn_kernels;

namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  std::call_once(g_encode_once, [] {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#ifdef ATTN_TRACE
// Trace buffer of the ATTN_TRACE build (attn_trace_configure); every launch
// of the forward kernel records into it.
uint2* g_trace = nullptr;
int g_trace_per_role = 0;
#endif

void set_trace(FwdArgs& a) {
#ifdef ATTN_TRACE
  a.trace = g_trace;
  a.trace_per_role = g_trace_per_role;
#else
  a.trace = nullptr;
  a.trace_per_role = 0;
#endif
}

// A bf16 tensor map over (dims[0] contiguous, dims[1..r-1] with element
// strides), box = {64, box_rows, 1, ...}, 128-byte swizzle.
// Tiled bf16 map with a 64-column inner box (SW128); box_rows rows along
// dimension box_rows_dim and, when box2_dim > 0, box2_rows along box2_dim.
attn_status make_map(CUtensorMap* m, const void* base, int rank, const uint64_t* dims, const int64_t* strides_el,
                     uint32_t box_rows, int box_rows_dim, uint32_t box2_rows = 1, int box2_dim = 0) {
  auto enc = encoder();
  if (!enc) return ATTN_ERR_CUDA;
  cuuint64_t gdim[5];
  cuuint64_t gstride[4];
  cuuint32_t box[5];
  cuuint32_t es[5];
  for (int i = 0; i < rank; ++i) {
    gdim[i] = dims[i];
    box[i] = 1;
    es[i] = 1;
    if (dims[i] == 0 || dims[i] > (1ull << 32)) return ATTN_ERR_UNSUPPORTED;
  }
  box[0] = 64;
  box[box_rows_dim] = box_rows;
  if (box2_dim > 0) box[box2_dim] = box2_rows;
  for (int i = 1; i < rank; ++i) {
    const int64_t b = strides_el[i - 1] * 2;
    if (b <= 0 || (b % 16) != 0 || b >= (1ll << 40)) return ATTN_ERR_UNSUPPORTED;
    gstride[i - 1] = static_cast<cuuint64_t>(b);
  }
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), gdim, gstride, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_UNSUPPORTED;
}

// The dynamic shared-memory opt-in is per device; remember which devices
// have it for each kernel instantiation.
template <int D, bool DECODE, int MOD, bool BM>
attn_status launch_fwd_mod(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mo,
                           const FwdArgs& a, int grid, cudaStream_t stream) {
  using L = Layout<D, DECODE>;
  static std::mutex mu;
  static uint64_t ready_mask = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ATTN_ERR_CUDA;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!(ready_mask & (1ull << dev))) {
      if (cudaFuncSetAttribute(attn_fwd_kernel<D, DECODE, MOD, BM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               L::kSmemBytes) != cudaSuccess)
        return ATTN_ERR_CUDA;
      ready_mask |= 1ull << dev;
    }
  }
  attn_fwd_kernel<D, DECODE, MOD, BM><<<grid, kThreads, L::kSmemBytes, stream>>>(mq, mk, mv, mo, a);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// One kernel per score mod, and (prefill) per "block mask given or not",
// keeps each instantiation's code small: code that runs once per work unit
// (setup, masked tiles, epilogue) is otherwise evicted from the instruction
// cache by the hot loop and refetched every unit.
template <int D, bool DECODE, bool BM>
attn_status launch_fwd_bm(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mo,
                          const FwdArgs& a, int grid, cudaStream_t stream) {
  switch (a.mod) {
    case MOD_SOFTCAP:
      return launch_fwd_mod<D, DECODE, MOD_SOFTCAP, BM>(mq, mk, mv, mo, a, grid, stream);
    case MOD_ALIBI:
      return launch_fwd_mod<D, DECODE, MOD_ALIBI, BM>(mq, mk, mv, mo, a, grid, stream);
    case MOD_RELU:
      if constexpr (DECODE)
        return ATTN_ERR_UNSUPPORTED;
      else
        return launch_fwd_mod<D, DECODE, MOD_RELU, BM>(mq, mk, mv, mo, a, grid, stream);
    default:
      return launch_fwd_mod<D, DECODE, MOD_NONE, BM>(mq, mk, mv, mo, a, grid, stream);
  }
}
template <int D, bool DECODE>
attn_status launch_fwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mo,
                       const FwdArgs& a, int grid, cudaStream_t stream) {
  if (!DECODE && a.bm_cls != nullptr) return launch_fwd_bm<D, DECODE, !DECODE>(mq, mk, mv, mo, a, grid, stream);
  return launch_fwd_bm<D, DECODE, false>(mq, mk, mv, mo, a, grid, stream);
}

// Streaming multiprocessors of the current device (persistent grid size).
int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

bool strides_ok(const int64_t* s, int n) {
  for (int i = 0; i < n; ++i)
    if (s[i] < 0 || (s[i] % 8) != 0) return false;
  return true;
}

// Element strides [b, s, h] of a [B, S, H, D] tensor reordered to the tensor
// map's (s, h, b) order. A size-1 dimension's stride is never used, so any
// value there is replaced by one the encoder accepts; a zero stride on a
// longer dimension (rows aliasing each other) is refused.
bool map_strides(const int64_t* bsh, const uint64_t* dims, int64_t* out) {
  const int64_t in[3] = {bsh[1], bsh[2], bsh[0]};
  for (int i = 0; i < 3; ++i) {
    if (dims[i + 1] == 1)
      out[i] = in[i] > 0 ? in[i] : 8;
    else if (in[i] > 0)
      out[i] = in[i];
    else
      return false;
  }
  return true;
}

attn_status check_mods(attn_mod_kind mod, float softcap, const float* alibi, int alibi_bstride, int Hq) {
  if (mod == ATTN_MOD_SOFTCAP && !(softcap > 0.f && std::isfinite(softcap))) return ATTN_ERR_INVALID_ARG;
  if (mod == ATTN_MOD_ALIBI && (alibi == nullptr || (alibi_bstride != 0 && alibi_bstride != Hq)))
    return ATTN_ERR_INVALID_ARG;
  if (mod != ATTN_MOD_NONE && mod != ATTN_MOD_SOFTCAP && mod != ATTN_MOD_ALIBI && mod != ATTN_MOD_RELU)
    return ATTN_ERR_INVALID_ARG;
  return ATTN_OK;
}

// Backward launches: the smem opt-in is per device and kernel.
template <typename K>
attn_status opt_in_smem(K kernel, int bytes, uint64_t& ready_mask, std::mutex& mu) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (!(ready_mask & (1ull << dev))) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
      return ATTN_ERR_CUDA;
    ready_mask |= 1ull << dev;
  }
  return ATTN_OK;
}

template <int D>
attn_status launch_bwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mdo,
                       attn_bwd_kernels::BwdArgs a, cudaStream_t st) {
  using namespace attn_bwd_kernels;
  using L = BLayout<D>;
  static std::mutex mu1, mu2;
  static uint64_t r1 = 0, r2 = 0;
  if (attn_status e = opt_in_smem(attn_bwd_dkdv_kernel<D>, L::kSmemBytes, r1, mu1)) return e;
  if (attn_status e = opt_in_smem(attn_bwd_dq_kernel<D>, L::kSmemBytes, r2, mu2)) return e;
  const int sms = sm_count();
  if (a.Skv > 0) {
    a.n_units = a.B * a.Hkv * a.n_pieces;
    attn_bwd_dkdv_kernel<D><<<a.n_units < sms ? a.n_units : sms, kBwdThreads, L::kSmemBytes, st>>>(mq, mk, mv, mdo,
                                                                                                    a);
    if (a.n_slots > 0)
      attn_bwd_dkdv_reduce_kernel<D><<<dim3(a.nK, a.B * a.Hkv, kTile * D / 8 / kReduceThreads), kReduceThreads, 0, st>>>(a);
  }
  a.n_units = a.B * a.Hq * a.nQ;
  attn_bwd_dq_kernel<D><<<a.n_units < sms ? a.n_units : sms, kBwdThreads, L::kSmemBytes, st>>>(mq, mk, mv, mdo, a);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// The dK/dV plan and workspace layout of a backward call: pieces per key
// tile under a cap chosen so that there are about two pieces per SM (the
// plan block on the device repeats the same integer arithmetic).
struct BwdPlan {
  int nQ, nK, g, mask, wl, wr, q_offset, cap, n_pieces, n_slots;
  size_t off_pieces, off_tiles, off_part, bytes;
};

bool bwd_plan(const attn_bwd_params* p, int sms, BwdPlan* out) {
  using namespace attn_bwd_kernels;
  if (!p || p->B < 0 || p->Sq < 0 || p->Skv < 0 || p->Hq <= 0 || p->Hkv <= 0 || p->Hq % p->Hkv != 0) return false;
  if (p->D != 64 && p->D != 128) return false;
  if (p->mask.kind != ATTN_MASK_NONE && p->mask.kind != ATTN_MASK_CAUSAL && p->mask.kind != ATTN_MASK_WINDOW)
    return false;
  BwdPlan& q = *out;
  q.g = p->Hq / p->Hkv;
  q.mask = p->mask.kind;
  q.q_offset = p->mask.kind == ATTN_MASK_NONE ? 0 : p->mask.q_offset;
  q.wl = p->mask.kind == ATTN_MASK_WINDOW ? (p->mask.window_left < 0 ? -1 : p->mask.window_left) : -1;
  q.wr = p->mask.kind == ATTN_MASK_CAUSAL
             ? 0
             : (p->mask.kind == ATTN_MASK_WINDOW ? (p->mask.window_right < 0 ? -1 : p->mask.window_right) : -1);
  q.nQ = (p->Sq + kTile - 1) / kTile;
  q.nK = (p->Skv + kTile - 1) / kTile;
  long long total = 0;
  int qlo;
  for (int t = 0; t < q.nK; ++t)
    total += kv_tile_steps(p->Sq, p->Skv, q.g, q.mask, q.wl, q.wr, q.q_offset, t, &qlo);
  total *= (long long)p->B * p->Hkv;
  const long long want = (total + 2LL * sms - 1) / (2LL * sms);
  q.cap = (int)(want < 4 ? 4 : (want > (1LL << 30) ? (1LL << 30) : want));
  long long np_sum = 0, slots = 0;
  for (int t = 0; t < q.nK; ++t) {
    const int np = kv_tile_pieces(kv_tile_steps(p->Sq, p->Skv, q.g, q.mask, q.wl, q.wr, q.q_offset, t, &qlo), q.cap);
    np_sum += np;
    slots += np > 1 ? np : 0;
  }
  if (np_sum * p->B * p->Hkv > 0x7fffffffLL || (long long)p->B * p->Hq * q.nQ > 0x7fffffffLL) return false;
  q.n_pieces = (int)np_sum;
  q.n_slots = (int)slots;
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  q.off_pieces = up((size_t)p->B * p->Hq * p->Sq * sizeof(float));
  q.off_tiles = q.off_pieces + up((size_t)q.n_pieces * 16);
  q.off_part = q.off_tiles + up((size_t)(q.nK > 0 ? q.nK : 1) * 8);
  q.bytes = q.off_part + (size_t)p->B * p->Hkv * q.n_slots * 2 * kTile * p->D * sizeof(float);
  return true;
}

}  // namespace

extern "C" {

size_t attn_bwd_workspace_bytes(const attn_bwd_params* p) {
  BwdPlan plan;
  if (!p || p->B <= 0 || p->Sq <= 0 || !bwd_plan(p, sm_count(), &plan)) return 0;
  return plan.bytes;
}

attn_status attn_bwd(const attn_bwd_params* p, void* workspace, size_t workspace_bytes, void* stream) {
  using namespace attn_bwd_kernels;
  if (!p) return ATTN_ERR_INVALID_ARG;
  if (p->B < 0 || p->Sq < 0 || p->Skv < 0 || p->Hq <= 0 || p->Hkv <= 0) return ATTN_ERR_INVALID_ARG;
  if (p->Hq % p->Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (p->D != 64 && p->D != 128) return ATTN_ERR_UNSUPPORTED;
  if (p->mask.kind != ATTN_MASK_NONE && p->mask.kind != ATTN_MASK_CAUSAL && p->mask.kind != ATTN_MASK_WINDOW)
    return p->mask.kind == ATTN_MASK_DOCUMENT ? ATTN_ERR_UNSUPPORTED : ATTN_ERR_INVALID_ARG;
  if (p->B == 0 || p->Sq == 0) return ATTN_OK;
  if (!p->q || !p->o || !p->dout || !p->lse || !p->dq || (p->Skv > 0 && (!p->k || !p->v || !p->dk || !p->dv)))
    return ATTN_ERR_INVALID_ARG;
  const void* ptrs[] = {p->q, p->k, p->v, p->o, p->dout, p->dq, p->dk, p->dv};
  for (const void* x : ptrs)
    if (x && !aligned16(x)) return ATTN_ERR_UNSUPPORTED;
  const int64_t* strides[] = {p->q_stride, p->k_stride, p->v_stride, p->o_stride,
                              p->do_stride, p->dq_stride, p->dk_stride, p->dv_stride};
  for (const int64_t* st : strides)
    if (!strides_ok(st, 3)) return ATTN_ERR_UNSUPPORTED;
  BwdPlan plan;
  if (!bwd_plan(p, sm_count(), &plan)) return ATTN_ERR_UNSUPPORTED;
  if (!workspace || !aligned16(workspace)) return ATTN_ERR_INVALID_ARG;
  if (workspace_bytes < plan.bytes) return ATTN_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);

  BwdArgs a{};
  a.B = p->B;
  a.Hq = p->Hq;
  a.Hkv = p->Hkv;
  a.Sq = p->Sq;
  a.Skv = p->Skv;
  a.g = plan.g;
  a.scale = p->scale > 0.f ? p->scale : 1.0f / std::sqrt(static_cast<float>(p->D));
  a.scale_log2 = a.scale * kLog2e;
  a.mask = plan.mask;
  a.q_offset = plan.q_offset;
  a.wl = plan.wl;
  a.wr = plan.wr;
  a.nQ = plan.nQ;
  a.nK = plan.nK;
  a.lse = p->lse;
  a.delta = reinterpret_cast<const float*>(ws);
  a.dq = static_cast<__nv_bfloat16*>(p->dq);
  a.dk = static_cast<__nv_bfloat16*>(p->dk);
  a.dv = static_cast<__nv_bfloat16*>(p->dv);
  a.dq_sb = p->dq_stride[0];
  a.dq_ss = p->dq_stride[1];
  a.dq_sh = p->dq_stride[2];
  a.dk_sb = p->dk_stride[0];
  a.dk_ss = p->dk_stride[1];
  a.dk_sh = p->dk_stride[2];
  a.dv_sb = p->dv_stride[0];
  a.dv_ss = p->dv_stride[1];
  a.dv_sh = p->dv_stride[2];
  a.pieces = reinterpret_cast<const int4*>(ws + plan.off_pieces);
  a.tiles = reinterpret_cast<const int2*>(ws + plan.off_tiles);
  a.part = reinterpret_cast<float*>(ws + plan.off_part);
  a.n_pieces = plan.n_pieces;
  a.n_slots = plan.n_slots;
  a.cap = plan.cap;
  a.status = p->status;

  // rowsum(dO o O) per (b, h, i); the extra last block writes the plan
  DeltaArgs da;
  da.o = static_cast<const __nv_bfloat16*>(p->o);
  da.dout = static_cast<const __nv_bfloat16*>(p->dout);
  da.o_sb = p->o_stride[0];
  da.o_ss = p->o_stride[1];
  da.o_sh = p->o_stride[2];
  da.do_sb = p->do_stride[0];
  da.do_ss = p->do_stride[1];
  da.do_sh = p->do_stride[2];
  da.B = p->B;
  da.Hq = p->Hq;
  da.Sq = p->Sq;
  da.D = p->D;
  da.delta = reinterpret_cast<float*>(ws);
  const int64_t rows = (int64_t)p->B * p->Hq * p->Sq;
  const int rows_per_block = 256 / (p->D / 8);
  const int64_t delta_blocks = (rows + rows_per_block - 1) / rows_per_block;
  if (delta_blocks + 1 > 0x7fffffffL) return ATTN_ERR_UNSUPPORTED;
  da.delta_blocks = (int)delta_blocks;
  da.plan = a;

  CUtensorMap mq, mk, mv, mdo;
  const uint64_t dq[4] = {(uint64_t)p->D, (uint64_t)p->Sq, (uint64_t)p->Hq, (uint64_t)p->B};
  const uint64_t dk[4] = {(uint64_t)p->D, (uint64_t)(p->Skv > 0 ? p->Skv : 1), (uint64_t)p->Hkv, (uint64_t)p->B};
  int64_t sq[3], sk[3], sv[3], sdo[3];
  if (!map_strides(p->q_stride, dq, sq) || !map_strides(p->do_stride, dq, sdo) ||
      (p->Skv > 0 && (!map_strides(p->k_stride, dk, sk) || !map_strides(p->v_stride, dk, sv))))
    return ATTN_ERR_UNSUPPORTED;
  if (p->Skv == 0) {
    for (int i = 0; i < 3; ++i) sk[i] = sv[i] = sq[i];
  }
  if (attn_status e = make_map(&mq, p->q, 4, dq, sq, kTile, 1)) return e;
  if (attn_status e = make_map(&mdo, p->dout, 4, dq, sdo, kTile, 1)) return e;
  // With Skv == 0 no key tile is ever loaded; the unused maps point at Q.
  if (attn_status e = make_map(&mk, p->Skv > 0 ? p->k : p->q, 4, p->Skv > 0 ? dk : dq, sk, kTile, 1)) return e;
  if (attn_status e = make_map(&mv, p->Skv > 0 ? p->v : p->q, 4, p->Skv > 0 ? dk : dq, sv, kTile, 1)) return e;
  delta_kernel<<<(unsigned)(delta_blocks + 1), kPlanThreads, 0, st>>>(da);
  return p->D == 128 ? launch_bwd<128>(mq, mk, mv, mdo, a, st) : launch_bwd<64>(mq, mk, mv, mdo, a, st);
}

attn_status attn_kvcache_update(const attn_kvcache_update_params* p, void* stream) {
  using namespace attn_kv_kernels;
  if (!p) return ATTN_ERR_INVALID_ARG;
  if (p->B < 0 || p->Snew < 0 || p->Hq < 0 || p->Hkv < 0 || p->page_size <= 0 || p->num_pages <= 0)
    return ATTN_ERR_INVALID_ARG;
  if (p->D != 64 && p->D != 128) return ATTN_ERR_UNSUPPORTED;
  const bool has_q = p->q != nullptr, has_kv = p->k_new != nullptr;
  if (has_kv != (p->v_new != nullptr) || (has_q && !p->q_out) || (has_kv && (!p->k_cache || !p->v_cache)))
    return ATTN_ERR_INVALID_ARG;
  if (!p->cache_seqlens) return ATTN_ERR_INVALID_ARG;
  if (p->block_table && p->block_table_stride <= 0) return ATTN_ERR_INVALID_ARG;
  if (p->rotary_cos || p->rotary_sin) {
    if (!p->rotary_cos || !p->rotary_sin || p->rotary_positions <= 0) return ATTN_ERR_INVALID_ARG;
    if (p->rotary_dim <= 0 || p->rotary_dim % 16 != 0 || p->rotary_dim > p->D) return ATTN_ERR_UNSUPPORTED;
  }
  const void* ptrs[] = {p->q, p->q_out, p->k_new, p->v_new, p->k_cache, p->v_cache};
  for (const void* x : ptrs)
    if (x && !aligned16(x)) return ATTN_ERR_UNSUPPORTED;
  const int64_t* strides[] = {p->q_stride, p->q_out_stride, p->k_new_stride, p->v_new_stride, p->cache_stride};
  for (const int64_t* st : strides)
    if (!strides_ok(st, 3)) return ATTN_ERR_UNSUPPORTED;
  if (p->B == 0) return ATTN_OK;
  KvUpdateArgs a{};
  a.q = static_cast<const __nv_bfloat16*>(p->q);
  a.q_sb = p->q_stride[0];
  a.q_ss = p->q_stride[1];
  a.q_sh = p->q_stride[2];
  a.q_out = static_cast<__nv_bfloat16*>(p->q_out);
  a.qo_sb = p->q_out_stride[0];
  a.qo_ss = p->q_out_stride[1];
  a.qo_sh = p->q_out_stride[2];
  a.k_new = static_cast<const __nv_bfloat16*>(p->k_new);
  a.v_new = static_cast<const __nv_bfloat16*>(p->v_new);
  a.kn_sb = p->k_new_stride[0];
  a.kn_ss = p->k_new_stride[1];
  a.kn_sh = p->k_new_stride[2];
  a.vn_sb = p->v_new_stride[0];
  a.vn_ss = p->v_new_stride[1];
  a.vn_sh = p->v_new_stride[2];
  a.k_cache = static_cast<__nv_bfloat16*>(p->k_cache);
  a.v_cache = static_cast<__nv_bfloat16*>(p->v_cache);
  a.c_sp = p->cache_stride[0];
  a.c_ss = p->cache_stride[1];
  a.c_sh = p->cache_stride[2];
  a.block_table = p->block_table;
  a.bt_stride = p->block_table_stride;
  a.cache_batch_idx = p->block_table ? nullptr : p->cache_batch_idx;
  a.seqlens = p->cache_seqlens;
  a.seqlens_out = p->seqlens_out;
  a.B = p->B;
  a.Snew = p->Snew;
  a.Hq = p->Hq;
  a.Hkv = p->Hkv;
  a.D = p->D;
  a.page_size = p->page_size;
  a.num_pages = p->num_pages;
  a.cos = p->rotary_cos;
  a.sin = p->rotary_sin;
  a.rot_dim = p->rotary_cos ? p->rotary_dim : 0;
  a.rot_positions = p->rotary_positions;
  a.interleaved = p->rotary_interleaved ? 1 : 0;
  a.status = p->status;
  const int64_t q_rows = has_q ? (int64_t)p->B * p->Snew * p->Hq : 0;
  const int64_t kv_rows = has_kv ? (int64_t)p->B * p->Snew * p->Hkv : 0;
  if (q_rows > 0x7fffffffL) return ATTN_ERR_UNSUPPORTED;
  a.q_rows = (int)q_rows;
  int64_t threads = (q_rows + kv_rows) * (p->D / 8);
  if (threads < p->B) threads = p->B;  // seqlens_out
  const int64_t blocks = (threads + 255) / 256;
  if (blocks > 0x7fffffffL) return ATTN_ERR_UNSUPPORTED;
  kvcache_update_kernel<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(a);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

const char* attn_status_str(attn_status s) {
  switch (s) {
    case ATTN_OK:
      return "ok";
    case ATTN_ERR_INVALID_ARG:
      return "invalid argument";
    case ATTN_ERR_UNSUPPORTED:
      return "unsupported configuration";
    case ATTN_ERR_CUDA:
      return "CUDA error";
    case ATTN_ERR_WORKSPACE:
      return "workspace too small";
  }
  return "unknown status";
}

size_t attn_block_mask_bytes(int Bm, int Hm, int Sq, int Skv, int blk_q, int blk_kv) {
  if (Bm <= 0 || Hm <= 0 || Sq <= 0 || Skv <= 0 || blk_q <= 0 || blk_kv <= 0) return 0;
  const size_t slices = (size_t)Bm * Hm;
  const size_t nQ = (Sq + blk_q - 1) / blk_q, nK = (Skv + blk_kv - 1) / blk_kv;
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  return up(slices * nQ * nK) + 2 * up(slices * nQ * 4) + 2 * up(slices * nQ * nK * 4) + up((size_t)Bm * nQ * 4) +
         up((size_t)Bm * Sq * 4) + up((size_t)Bm * 4);
}

attn_status attn_block_mask_layout(void* buf, size_t buf_bytes, int Bm, int Hm, int Sq, int Skv, int blk_q,
                                   int blk_kv, attn_block_mask* out) {
  if (!out || !buf || !aligned16(buf)) return ATTN_ERR_INVALID_ARG;
  const size_t need = attn_block_mask_bytes(Bm, Hm, Sq, Skv, blk_q, blk_kv);
  if (need == 0) return ATTN_ERR_INVALID_ARG;
  if (buf_bytes < need) return ATTN_ERR_WORKSPACE;
  const size_t slices = (size_t)Bm * Hm;
  const size_t nQ = (Sq + blk_q - 1) / blk_q, nK = (Skv + blk_kv - 1) / blk_kv;
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  uint8_t* p = static_cast<uint8_t*>(buf);
  out->Bm = Bm;
  out->Hm = Hm;
  out->Sq = Sq;
  out->Skv = Skv;
  out->blk_q = blk_q;
  out->blk_kv = blk_kv;
  out->n_q_tiles = static_cast<int>(nQ);
  out->n_kv_tiles = static_cast<int>(nK);
  out->cls = p;
  p += up(slices * nQ * nK);
  out->part_cnt = reinterpret_cast<int32_t*>(p);
  p += up(slices * nQ * 4);
  out->full_cnt = reinterpret_cast<int32_t*>(p);
  p += up(slices * nQ * 4);
  out->part_idx = reinterpret_cast<int32_t*>(p);
  p += up(slices * nQ * nK * 4);
  out->full_idx = reinterpret_cast<int32_t*>(p);
  p += up(slices * nQ * nK * 4);
  out->row_order = reinterpret_cast<int32_t*>(p);
  p += up((size_t)Bm * nQ * 4);
  out->doc_start = reinterpret_cast<int32_t*>(p);
  p += up((size_t)Bm * Sq * 4);
  out->doc_sorted = reinterpret_cast<int32_t*>(p);
  return ATTN_OK;
}

attn_status attn_build_block_mask(const attn_mask_spec* spec, const attn_block_mask* out, void* stream) {
  if (!spec || !out) return ATTN_ERR_INVALID_ARG;
  if (out->Bm <= 0 || out->Hm <= 0 || out->Sq <= 0 || out->Skv <= 0 || out->blk_q <= 0 || out->blk_kv <= 0)
    return ATTN_ERR_INVALID_ARG;
  if (out->blk_q % 16 || out->blk_kv % 16 || out->blk_q > 1024 || out->blk_kv > 1024) return ATTN_ERR_UNSUPPORTED;
  if (out->Bm > 65535 || (long)out->Bm * out->Hm * ((out->Sq + out->blk_q - 1) / out->blk_q) > 0x7fffffffL)
    return ATTN_ERR_UNSUPPORTED;
  if (out->n_q_tiles != (out->Sq + out->blk_q - 1) / out->blk_q ||
      out->n_kv_tiles != (out->Skv + out->blk_kv - 1) / out->blk_kv)
    return ATTN_ERR_INVALID_ARG;
  if (!out->cls || !out->part_cnt || !out->part_idx || !out->full_cnt || !out->full_idx || !out->row_order)
    return ATTN_ERR_INVALID_ARG;
  if (spec->kind == ATTN_MASK_DOCUMENT && (!out->doc_start || !out->doc_sorted)) return ATTN_ERR_INVALID_ARG;
  if (spec->kind < ATTN_MASK_NONE || spec->kind > ATTN_MASK_DOCUMENT) return ATTN_ERR_INVALID_ARG;
  if (spec->kind == ATTN_MASK_DOCUMENT) {
    if (!spec->doc_id || out->Sq != out->Skv || spec->q_offset != 0) return ATTN_ERR_INVALID_ARG;
    if (spec->doc_batch_stride < 0 || (spec->doc_batch_stride > 0 && spec->doc_batch_stride < out->Sq))
      return ATTN_ERR_INVALID_ARG;
  }
  MaskArgs a;
  a.kind = spec->kind;
  a.wl = spec->kind == ATTN_MASK_CAUSAL ? -1 : spec->window_left;
  a.wr = spec->kind == ATTN_MASK_CAUSAL ? 0 : spec->window_right;
  a.q_offset = spec->kind == ATTN_MASK_NONE ? 0 : spec->q_offset;
  a.doc_id = spec->doc_id;
  a.doc_bstride = spec->kind == ATTN_MASK_DOCUMENT ? spec->doc_batch_stride : 0;
  a.Bm = out->Bm;
  a.Hm = out->Hm;
  a.Sq = out->Sq;
  a.Skv = out->Skv;
  a.blk_q = out->blk_q;
  a.blk_kv = out->blk_kv;
  a.nQ = out->n_q_tiles;
  a.nK = out->n_kv_tiles;
  a.cls = out->cls;
  a.part_cnt = out->part_cnt;
  a.part_idx = out->part_idx;
  a.full_cnt = out->full_cnt;
  a.full_idx = out->full_idx;
  a.row_order = out->row_order;
  a.doc_start = out->doc_start;
  a.doc_sorted = out->doc_sorted;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // Pass 1 classifies head slice 0 of every batch slice (the mask kinds do not
  // depend on the head); pass 2 copies it to the other head slices and builds
  // every slice's lists. A mask that does not depend on the batch either
  // (no per-batch document rows) is classified once and copied.
  const int b_class = (a.kind == ATTN_MASK_DOCUMENT && a.doc_bstride > 0) ? a.Bm : 1;
  if (a.kind == ATTN_MASK_DOCUMENT) {
    const size_t smem = (size_t)kKvPerCta * a.blk_kv * sizeof(int);
    classify_doc_kernel<<<dim3(a.nQ, (a.nK + kKvPerCta - 1) / kKvPerCta, b_class), kMaskThreads, smem, st>>>(a);
  } else {
    const int64_t tiles = (int64_t)a.nQ * a.nK;
    classify_range_kernel<<<(unsigned)((tiles + 255) / 256), 256, 0, st>>>(a);
  }
  compact_lists_kernel<<<dim3(a.nQ, a.Bm * a.Hm), 32, 0, st>>>(a, b_class);
  row_order_kernel<<<a.Bm, kOrderThreads, 0, st>>>(a);
  if (a.kind == ATTN_MASK_DOCUMENT) doc_runs_kernel<<<a.Bm, kRunThreads, 0, st>>>(a);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

attn_status attn_fwd(const attn_fwd_params* p, void* stream) {
  if (!p) return ATTN_ERR_INVALID_ARG;
  if (p->B < 0 || p->Sq < 0 || p->Skv < 0 || p->Hq <= 0 || p->Hkv <= 0) return ATTN_ERR_INVALID_ARG;
  if (p->Hq % p->Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (p->D != 64 && p->D != 128) return ATTN_ERR_UNSUPPORTED;
  if (p->B == 0 || p->Sq == 0) return ATTN_OK;
  if (!p->q || !p->o || (p->Skv > 0 && (!p->k || !p->v))) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(p->q) || !aligned16(p->o) || (p->k && !aligned16(p->k)) || (p->v && !aligned16(p->v)))
    return ATTN_ERR_UNSUPPORTED;
  if (!strides_ok(p->q_stride, 3) || !strides_ok(p->k_stride, 3) || !strides_ok(p->v_stride, 3) ||
      !strides_ok(p->o_stride, 3))
    return ATTN_ERR_UNSUPPORTED;
  if (p->mask.kind < ATTN_MASK_NONE || p->mask.kind > ATTN_MASK_DOCUMENT) return ATTN_ERR_INVALID_ARG;
  if (attn_status st = check_mods(p->mod, p->softcap, p->alibi_slopes, p->alibi_batch_stride, p->Hq)) return st;
  const int nQ = (p->Sq + kRows - 1) / kRows;
  const int nK = (p->Skv + kKeys - 1) / kKeys;
  if (p->mask.kind == ATTN_MASK_DOCUMENT) {
    if (!p->mask.doc_id || p->Sq != p->Skv || p->mask.q_offset != 0 || !p->block_mask) return ATTN_ERR_INVALID_ARG;
    if (p->mask.doc_batch_stride < 0 || (p->mask.doc_batch_stride > 0 && p->mask.doc_batch_stride < p->Sq))
      return ATTN_ERR_INVALID_ARG;
    // rows are read as int4 by the kernel
    if (!aligned16(p->mask.doc_id) || p->mask.doc_batch_stride % 4) return ATTN_ERR_UNSUPPORTED;
  }
  if (p->block_mask) {
    const attn_block_mask* bm = p->block_mask;
    // 128 x 128 tables, or 256 x 128: one table row per two-subtile CTA
    if ((bm->blk_q != kRows && bm->blk_q != 2 * kRows) || bm->blk_kv != kKeys || bm->Sq != p->Sq ||
        bm->Skv != p->Skv || !bm->cls || bm->n_q_tiles != (p->Sq + bm->blk_q - 1) / bm->blk_q ||
        bm->n_kv_tiles != nK || !bm->part_cnt || !bm->part_idx || !bm->full_cnt || !bm->full_idx)
      return ATTN_ERR_INVALID_ARG;
    if ((bm->Bm != 1 && bm->Bm != p->B) || (bm->Hm != 1 && bm->Hm != p->Hq)) return ATTN_ERR_INVALID_ARG;
    if (p->mask.kind == ATTN_MASK_DOCUMENT && (!bm->doc_start || !bm->doc_sorted)) return ATTN_ERR_INVALID_ARG;
  }

  FwdArgs a{};
  a.B = p->B;
  a.Hq = p->Hq;
  a.Hkv = p->Hkv;
  a.Sq = p->Sq;
  a.Skv = p->Skv;
  a.g = p->Hq / p->Hkv;
  a.scale = p->scale > 0.f ? p->scale : 1.0f / std::sqrt(static_cast<float>(p->D));
  a.scale_log2 = a.scale * kLog2e;
  a.mask = p->mask.kind;
  switch (p->mask.kind) {
    case ATTN_MASK_NONE:
      a.wl = a.wr = -1;
      a.q_offset = 0;
      break;
    case ATTN_MASK_CAUSAL:
      a.wl = -1;
      a.wr = 0;
      a.q_offset = p->mask.q_offset;
      break;
    case ATTN_MASK_WINDOW:
      a.wl = p->mask.window_left < 0 ? -1 : p->mask.window_left;
      a.wr = p->mask.window_right < 0 ? -1 : p->mask.window_right;
      a.q_offset = p->mask.q_offset;
      break;
    default:
      a.wl = -1;
      a.wr = 0;
      a.q_offset = 0;
  }
  a.doc_id = p->mask.doc_id;
  a.doc_bstride = p->mask.kind == ATTN_MASK_DOCUMENT ? p->mask.doc_batch_stride : 0;
  a.bm_cls = p->block_mask ? p->block_mask->cls : nullptr;
  if (p->block_mask) {
    a.bm_Bm = p->block_mask->Bm;
    a.bm_Hm = p->block_mask->Hm;
    a.bm_rows = p->block_mask->blk_q;
    a.bm_nQ = p->block_mask->n_q_tiles;
    a.bm_row_order = p->block_mask->row_order;
    a.bm_doc_start = p->block_mask->doc_start;
    a.bm_doc_sorted = p->block_mask->doc_sorted;
    a.bm_part_cnt = p->block_mask->part_cnt;
    a.bm_part_idx = p->block_mask->part_idx;
    a.bm_full_cnt = p->block_mask->full_cnt;
    a.bm_full_idx = p->block_mask->full_idx;
  }
  a.nQ = nQ;
  a.nK = nK;
  a.mod = p->mod;
  a.softcap = p->softcap;
  a.softcap_k1 = p->softcap > 0.f ? a.scale / p->softcap : 0.f;
  a.alibi = p->alibi_slopes;
  a.alibi_bstride = p->alibi_batch_stride;
  a.o = static_cast<__nv_bfloat16*>(p->o);
  a.o_sb = p->o_stride[0];
  a.o_ss = p->o_stride[1];
  a.o_sh = p->o_stride[2];
  a.lse = p->lse;
  a.status = p->status;
  a.pair_heads = (a.g % 2 == 0) ? 1 : 0;
  a.n_row_units = a.pair_heads ? nQ : (nQ + 1) / 2;
  // a 256-row table in the paired-head layout: each table row is two units
  // (the second of an odd last row is empty)
  if (p->block_mask && a.pair_heads && a.bm_rows == 2 * kRows) a.n_row_units = 2 * a.bm_nQ;

  CUtensorMap mq, mk, mv, mo;
  const uint64_t dq[4] = {(uint64_t)p->D, (uint64_t)p->Sq, (uint64_t)p->Hq, (uint64_t)p->B};
  // Skv == 0: every row is fully masked; the maps are never read (no tile is visited).
  const uint64_t dk[4] = {(uint64_t)p->D, (uint64_t)(p->Skv > 0 ? p->Skv : 1), (uint64_t)p->Hkv, (uint64_t)p->B};
  int64_t sq[3], sk[3], sv[3], so[3];
  if (!map_strides(p->q_stride, dq, sq) || !map_strides(p->k_stride, dk, sk) || !map_strides(p->v_stride, dk, sv) ||
      !map_strides(p->o_stride, dq, so))
    return ATTN_ERR_UNSUPPORTED;
  if (attn_status st = make_map(&mq, p->q, 4, dq, sq, kRows, 1)) return st;
  // With Skv == 0 nothing is read from K / V; the unused maps point at Q.
  if (attn_status st = make_map(&mk, p->Skv > 0 ? p->k : p->q, 4, dk, sk, kKeys, 1)) return st;
  if (attn_status st = make_map(&mv, p->Skv > 0 ? p->v : p->q, 4, dk, sv, kKeys, 1)) return st;
  // O is written in 32-row boxes, one per softmax warp.
  if (attn_status st = make_map(&mo, p->o, 4, dq, so, 32, 1)) return st;

  set_trace(a);
  const int HU = a.pair_heads ? a.Hq / 2 : a.Hq;
  const long units = (long)a.B * HU * a.n_row_units;
  if (units <= 0 || units > 0x7fffffffL) return ATTN_ERR_UNSUPPORTED;
  a.n_units = (int)units;
  const long grid = units < sm_count() ? units : sm_count();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return p->D == 128 ? launch_fwd<128, false>(mq, mk, mv, mo, a, (int)grid, s)
                     : launch_fwd<64, false>(mq, mk, mv, mo, a, (int)grid, s);
}

int attn_decode_num_splits(int B, int Hq, int Hkv, int max_seqlen, int num_splits) {
  if (B <= 0 || Hkv <= 0 || Hq <= 0 || max_seqlen <= 0) return 1;
  const int tiles = (max_seqlen + kKeys - 1) / kKeys;
  if (num_splits > 0) return num_splits < tiles ? num_splits : tiles;
  // Pick the split count that minimises (waves of CTAs) x (tiles per split +
  // a fixed per-unit cost), favouring fewer splits on ties (less partial
  // traffic). The fixed cost (Q load, pipeline fill, merge and partial
  // write) is worth about ten key tiles on B200: for 32 sequences of 32768
  // tokens, one wave of 4 splits (128 units) measured 5371 GB/s against
  // 4746 GB/s for two waves of 9 splits and 4043 GB/s for 10.
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (sms <= 0) sms = 148;
  const long units = (long)B * Hkv;
  int best = 1;
  long best_cost = -1;
  for (int n = 1; n <= tiles && n <= 256; ++n) {
    const long waves = (units * n + sms - 1) / sms;
    const long per = (tiles + n - 1) / n;
    const long cost = waves * (per + 10);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = n;
    }
  }
  return best;
}

size_t attn_decode_workspace_bytes(int B, int Hq, int D, int num_splits) {
  if (B <= 0 || Hq <= 0 || D <= 0 || num_splits <= 0) return 0;
  const size_t rows = (size_t)B * Hq * num_splits;
  const size_t o_bytes = (rows * D * sizeof(float) + 255) & ~size_t(255);
  return o_bytes + rows * sizeof(float);
}

static attn_status launch_combine(const CombineArgs& c, int D, cudaStream_t s) {
  const int warps = 8;
  const int grid = (c.rows + warps - 1) / warps;
  if (D == 128)
    lse_combine_kernel<128><<<grid, warps * 32, 0, s>>>(c);
  else
    lse_combine_kernel<64><<<grid, warps * 32, 0, s>>>(c);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

attn_status attn_decode(const attn_decode_params* p, void* workspace, size_t workspace_bytes, void* stream) {
  if (!p) return ATTN_ERR_INVALID_ARG;
  if (p->B < 0 || p->Hq <= 0 || p->Hkv <= 0 || p->page_size <= 0 || p->num_pages <= 0) return ATTN_ERR_INVALID_ARG;
  if (p->Hq % p->Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (p->D != 64 && p->D != 128) return ATTN_ERR_UNSUPPORTED;
  const int q_len = p->q_len > 1 ? p->q_len : 1;
  const bool paged = p->block_table != nullptr;
  if (p->q_len < 0) return ATTN_ERR_INVALID_ARG;
  if ((p->Hq / p->Hkv) * q_len > kRows) return ATTN_ERR_UNSUPPORTED;
  if (paged && (p->page_size % 16 != 0 || (p->page_size < kKeys && kKeys % p->page_size != 0) ||
                (p->page_size > kKeys && p->page_size % kKeys != 0)))
    return ATTN_ERR_UNSUPPORTED;
  if (p->B == 0) return ATTN_OK;
  if (!p->q || !p->k_cache || !p->v_cache || !p->cache_seqlens || !p->o) return ATTN_ERR_INVALID_ARG;
  if (p->max_seqlen <= 0 || (paged && p->block_table_stride <= 0)) return ATTN_ERR_INVALID_ARG;
  if ((long)(paged ? p->block_table_stride : 1) * p->page_size < p->max_seqlen) return ATTN_ERR_INVALID_ARG;
  if (q_len > 1 && (p->q_token_stride <= 0 || p->o_token_stride <= 0 || (p->q_token_stride % 8) != 0))
    return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(p->q) || !aligned16(p->k_cache) || !aligned16(p->v_cache) || !aligned16(p->o))
    return ATTN_ERR_UNSUPPORTED;
  if (!strides_ok(p->q_stride, 2) || !strides_ok(p->cache_stride, 3) || !strides_ok(p->o_stride, 2))
    return ATTN_ERR_UNSUPPORTED;
  if (attn_status st = check_mods(p->mod, p->softcap, p->alibi_slopes, p->alibi_batch_stride, p->Hq)) return st;
  if (p->mod == ATTN_MOD_RELU) return ATTN_ERR_UNSUPPORTED;  // split partials assume normalised rows
  const int splits = attn_decode_num_splits(p->B, p->Hq, p->Hkv, p->max_seqlen, p->num_splits);
  const size_t need = attn_decode_workspace_bytes(p->B, p->Hq * q_len, p->D, splits);
  if (!workspace || !aligned16(workspace)) return ATTN_ERR_INVALID_ARG;
  if (workspace_bytes < need) return ATTN_ERR_WORKSPACE;

  FwdArgs a{};
  a.B = p->B;
  a.Hq = p->Hq;
  a.Hkv = p->Hkv;
  a.g = p->Hq / p->Hkv;
  a.scale = p->scale > 0.f ? p->scale : 1.0f / std::sqrt(static_cast<float>(p->D));
  a.scale_log2 = a.scale * kLog2e;
  a.mask = MASK_NONE;
  a.wl = a.wr = -1;
  a.mod = p->mod;
  a.softcap = p->softcap;
  a.softcap_k1 = p->softcap > 0.f ? a.scale / p->softcap : 0.f;
  a.alibi = p->alibi_slopes;
  a.alibi_bstride = p->alibi_batch_stride;
  a.status = p->status;
  a.block_table = p->block_table;
  a.cache_batch_idx = paged ? nullptr : p->cache_batch_idx;
  a.bt_stride = paged ? p->block_table_stride : 1;
  a.seqlens = p->cache_seqlens;
  a.page_size = p->page_size;
  a.num_pages = p->num_pages;
  a.box_rows = (paged && p->page_size < kKeys) ? p->page_size : kKeys;
  a.q_len = q_len;
  a.q_causal = q_len > 1 && p->causal ? 1 : 0;
  const int g = p->Hq / p->Hkv;
  const int tok_box = kRows / g;  // >= q_len
  a.q_bytes = (q_len > 1 ? g * tok_box : kRows) * p->D * 2;
  const int tiles = (p->max_seqlen + kKeys - 1) / kKeys;
  a.n_splits = splits;
  a.tiles_per_split = (tiles + splits - 1) / splits;
  a.max_seqlen = p->max_seqlen;
  const size_t rows = (size_t)p->B * q_len * p->Hq * splits;
  a.part_o = static_cast<float*>(workspace);
  a.part_lse = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + ((rows * p->D * 4 + 255) & ~size_t(255)));

  CUtensorMap mq, mk, mv;
  const uint64_t dq[3] = {(uint64_t)p->D, (uint64_t)p->Hq, (uint64_t)p->B};
  const int64_t sq[2] = {p->q_stride[1] > 0 ? p->q_stride[1] : 8, p->q_stride[0] > 0 ? p->q_stride[0] : 8};
  const uint64_t dc[4] = {(uint64_t)p->D, (uint64_t)p->Hkv, (uint64_t)p->page_size, (uint64_t)p->num_pages};
  const int64_t sc[3] = {p->cache_stride[2] > 0 ? p->cache_stride[2] : 8, p->cache_stride[1],
                         p->cache_stride[0]};
  if (q_len > 1) {
    // dims (D, g, Hkv, q_len, B), box (64, g, 1, 128 / g, 1): token i's heads land at rows i*g ..
    const uint64_t dq5[5] = {(uint64_t)p->D, (uint64_t)g, (uint64_t)p->Hkv, (uint64_t)q_len, (uint64_t)p->B};
    const int64_t sh = p->q_stride[1] > 0 ? p->q_stride[1] : 8;
    const int64_t sq5[4] = {sh, sh * g, p->q_token_stride, p->q_stride[0] > 0 ? p->q_stride[0] : 8};
    if (attn_status st = make_map(&mq, p->q, 5, dq5, sq5, (uint32_t)g, 1, (uint32_t)tok_box, 3)) return st;
  } else if (attn_status st = make_map(&mq, p->q, 3, dq, sq, kRows, 1)) {
    return st;
  }
  if (attn_status st = make_map(&mk, p->k_cache, 4, dc, sc, (uint32_t)a.box_rows, 2)) return st;
  if (attn_status st = make_map(&mv, p->v_cache, 4, dc, sc, (uint32_t)a.box_rows, 2)) return st;

  set_trace(a);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const long units = (long)p->B * p->Hkv * splits;
  if (units > 0x7fffffffL) return ATTN_ERR_UNSUPPORTED;
  a.n_units = (int)units;
  const long grid = units < sm_count() ? units : sm_count();
  // Decode writes fp32 partials with plain stores; its output map is unused.
  attn_status st = p->D == 128 ? launch_fwd<128, true>(mq, mk, mv, mq, a, (int)grid, s)
                               : launch_fwd<64, true>(mq, mk, mv, mq, a, (int)grid, s);
  if (st != ATTN_OK) return st;
  CombineArgs c;
  c.o_parts = a.part_o;
  c.lse_parts = a.part_lse;
  c.rows = p->B * q_len * p->Hq;
  c.n = splits;
  c.D = p->D;
  c.rows_per_b = q_len * p->Hq;
  c.heads = p->Hq;
  c.o = static_cast<__nv_bfloat16*>(p->o);
  c.o_sb = p->o_stride[0];
  c.o_st = q_len > 1 ? p->o_token_stride : 0;
  c.o_sh = p->o_stride[1];
  c.lse = p->lse;
  return launch_combine(c, p->D, s);
}

attn_status attn_lse_combine(const float* o_parts, const float* lse_parts, int rows, int n_splits, int D, void* o,
                             int64_t o_row_stride, float* lse, void* stream) {
  if (rows < 0 || n_splits <= 0 || (D != 64 && D != 128)) return rows < 0 || n_splits <= 0 ? ATTN_ERR_INVALID_ARG
                                                                                          : ATTN_ERR_UNSUPPORTED;
  if (rows == 0) return ATTN_OK;
  if (!o_parts || !lse_parts || !o) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(o_parts) || (reinterpret_cast<uintptr_t>(o) & 7u) || o_row_stride < D || (o_row_stride % 4))
    return ATTN_ERR_UNSUPPORTED;
  CombineArgs c;
  c.o_parts = o_parts;
  c.lse_parts = lse_parts;
  c.rows = rows;
  c.n = n_splits;
  c.D = D;
  c.rows_per_b = rows;
  c.heads = rows > 0 ? rows : 1;
  c.o = static_cast<__nv_bfloat16*>(o);
  c.o_sb = 0;
  c.o_st = 0;
  c.o_sh = o_row_stride;
  c.lse = lse;
  return launch_combine(c, D, static_cast<cudaStream_t>(stream));
}

#ifdef ATTN_TRACE
// Trace builds only: every later forward launch appends cycle records to buf
// (device memory, grid CTAs x 10 roles x per_role uint2 records; the caller
// zeroes it). buf = NULL turns tracing off.
attn_status attn_trace_configure(void* buf, int per_role) {
  if (buf != nullptr && per_role <= 0) return ATTN_ERR_INVALID_ARG;
  g_trace = static_cast<uint2*>(buf);
  g_trace_per_role = buf ? per_role : 0;
  return ATTN_OK;
}
#endif

}  // extern "C"
