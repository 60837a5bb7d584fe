// aux_kernels.cuh - CUDA-core kernels around the attention forward:
//   * block-mask builder (FlexAttention create_block_mask equivalent)
//   * LSE combine of split-KV partial results
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

namespace attn_kernels {

struct MaskArgs {
  int kind, wl, wr, q_offset;
  const int32_t* doc_id;
  int Sq, Skv, blk_q, blk_kv, nQ, nK;
  uint8_t* cls;
  int32_t *part_cnt, *part_idx, *full_cnt, *full_idx;
};

// Block-mask build, pass 1: classify tiles. CTA (q-tile, group of kKvPerCta
// kv-tiles); each thread evaluates its query rows against every in-range key
// of a tile (stopping early once it has seen both an allowed and a masked
// pair), then block votes give "any allowed" and "all allowed".
constexpr int kMaskThreads = 128;
constexpr int kKvPerCta = 8;

__device__ __forceinline__ bool pair_allowed(const MaskArgs& a, long q_pos, int j, int doc_i, int doc_j) {
  switch (a.kind) {
    case 0:
      return true;
    case 1:
      return (long)j <= q_pos;
    case 2:
      return (a.wl < 0 || q_pos - j <= a.wl) && (a.wr < 0 || (long)j - q_pos <= a.wr);
    default:
      return (long)j <= q_pos && doc_j == doc_i;
  }
}

__global__ void __launch_bounds__(kMaskThreads) classify_tiles_kernel(const MaskArgs a) {
  extern __shared__ int doc_k[];  // [kKvPerCta * blk_kv] key doc ids (document masks)
  const int qt = blockIdx.x;
  const int kt0 = blockIdx.y * kKvPerCta;
  const int kt1 = min(kt0 + kKvPerCta, a.nK);
  const int q0 = qt * a.blk_q;
  const int rows = min(a.blk_q, a.Sq - q0);
  const bool is_doc = a.kind == 3;
  if (is_doc) {
    const int k_first = kt0 * a.blk_kv, k_end = min(kt1 * a.blk_kv, a.Skv);
    for (int c = threadIdx.x; c < k_end - k_first; c += blockDim.x) doc_k[c] = a.doc_id[k_first + c];
  }
  __syncthreads();
  for (int kt = kt0; kt < kt1; ++kt) {
    const int k0 = kt * a.blk_kv;
    const int cols = min(a.blk_kv, a.Skv - k0);
    const int* dk = doc_k + (kt - kt0) * a.blk_kv;
    bool any = false, all = true;
    for (int r = threadIdx.x; r < rows && (all || !any); r += blockDim.x) {
      const long q_pos = (long)(q0 + r) + a.q_offset;
      const int di = is_doc ? a.doc_id[q0 + r] : 0;
      for (int c = 0; c < cols; ++c) {
        const bool ok = pair_allowed(a, q_pos, k0 + c, di, is_doc ? dk[c] : 0);
        any |= ok;
        all &= ok;
        if (any && !all) break;
      }
    }
    const int any_b = __syncthreads_or(any);
    const int all_b = __syncthreads_and(all);
    if (threadIdx.x == 0) a.cls[(int64_t)qt * a.nK + kt] = any_b ? (all_b ? 2 : 1) : 0;
  }
}

// Pass 2: one warp per q-tile compacts the class row into the ascending
// partial and full lists with ballots.
__global__ void __launch_bounds__(32) compact_lists_kernel(const MaskArgs a) {
  const int qt = blockIdx.x;
  const int lane = threadIdx.x;
  const uint8_t* row = a.cls + (int64_t)qt * a.nK;
  int np = 0, nf = 0;
  for (int k0 = 0; k0 < a.nK; k0 += 32) {
    const int kt = k0 + lane;
    const uint8_t c = kt < a.nK ? row[kt] : 0;
    const unsigned mp = __ballot_sync(0xffffffffu, c == 1);
    const unsigned mf = __ballot_sync(0xffffffffu, c == 2);
    const unsigned below = (1u << lane) - 1u;
    if (c == 1) a.part_idx[(int64_t)qt * a.nK + np + __popc(mp & below)] = kt;
    if (c == 2) a.full_idx[(int64_t)qt * a.nK + nf + __popc(mf & below)] = kt;
    np += __popc(mp);
    nf += __popc(mf);
  }
  if (lane == 0) {
    a.part_cnt[qt] = np;
    a.full_cnt[qt] = nf;
  }
}

// One warp per output row: lse = ln sum_i exp(lse_i); o = sum_i exp(lse_i - lse) o_i.
struct CombineArgs {
  const float* o_parts;    // [rows][n][D]
  const float* lse_parts;  // [rows][n]
  int rows, n, D;
  int rows_per_b;          // rows are (b, h) with h < rows_per_b
  __nv_bfloat16* o;
  int64_t o_sb, o_sh;      // element strides of the output rows (b, h)
  float* lse;              // [rows] or nullptr
};

template <int D>
__global__ void __launch_bounds__(256) lse_combine_kernel(const CombineArgs a) {
  const int row = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (row >= a.rows) return;
  const float* lp = a.lse_parts + (int64_t)row * a.n;
  const float NEG_INF = -__int_as_float(0x7f800000);
  float mx = NEG_INF;
  for (int i = lane; i < a.n; i += 32) mx = fmaxf(mx, lp[i]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  float sum = 0.f;
  if (mx != NEG_INF)
    for (int i = lane; i < a.n; i += 32) sum += expf(lp[i] - mx);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  const float lse = mx == NEG_INF ? NEG_INF : mx + logf(sum);
  constexpr int V = D / 32;  // elements per lane
  float acc[V];
#pragma unroll
  for (int j = 0; j < V; ++j) acc[j] = 0.f;
  if (mx != NEG_INF) {
    const float* op = a.o_parts + (int64_t)row * a.n * D + lane * V;
    for (int i = 0; i < a.n; ++i) {
      const float li = lp[i];
      if (li == NEG_INF) continue;
      const float wgt = expf(li - lse);
      if constexpr (V == 4) {
        const float4 f = *reinterpret_cast<const float4*>(op + (int64_t)i * D);
        acc[0] += wgt * f.x;
        acc[1] += wgt * f.y;
        acc[2] += wgt * f.z;
        acc[3] += wgt * f.w;
      } else {
        const float2 f = *reinterpret_cast<const float2*>(op + (int64_t)i * D);
        acc[0] += wgt * f.x;
        acc[1] += wgt * f.y;
      }
    }
  }
  const int b = row / a.rows_per_b, h = row % a.rows_per_b;
  __nv_bfloat16* dst = a.o + (int64_t)b * a.o_sb + (int64_t)h * a.o_sh + lane * V;
  if constexpr (V == 4) {
    __nv_bfloat162 p0 = __floats2bfloat162_rn(acc[0], acc[1]);
    __nv_bfloat162 p1 = __floats2bfloat162_rn(acc[2], acc[3]);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t*>(&p0);
    u.y = *reinterpret_cast<uint32_t*>(&p1);
    *reinterpret_cast<uint2*>(dst) = u;
  } else {
    *reinterpret_cast<__nv_bfloat162*>(dst) = __floats2bfloat162_rn(acc[0], acc[1]);
  }
  if (lane == 0 && a.lse != nullptr) a.lse[row] = lse;
}

}  // namespace attn_kernels
