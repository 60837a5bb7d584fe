// kvcache_kernel.cuh - in-place kv-cache update with rotary embedding
// (attn_kvcache_update): the k / v / rotary / cache_batch_idx / block_table
// part of flash_attn_with_kvcache (FlashAttention overview, "Examples").
//
// One thread per 8-element (16-byte) chunk of a head row. Rows are the new
// tokens' query heads (rotated, to q_out) and KV heads (k rotated, v copied,
// both to the cache). A rotary pair lies inside one chunk for the interleaved
// layout; for the half layout the thread also loads the partner chunk
// rotary_dim / 16 chunks away. HBM-bound: every byte is read once and
// written once.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

namespace attn_kv_kernels {

enum : int { KV_BAD_PAGE = 2, KV_BAD_LEN = 4 };

struct KvUpdateArgs {
  const __nv_bfloat16* q;
  int64_t q_sb, q_ss, q_sh;
  __nv_bfloat16* q_out;
  int64_t qo_sb, qo_ss, qo_sh;
  const __nv_bfloat16 *k_new, *v_new;
  int64_t kn_sb, kn_ss, kn_sh, vn_sb, vn_ss, vn_sh;
  __nv_bfloat16 *k_cache, *v_cache;
  int64_t c_sp, c_ss, c_sh;  // page (row), slot (position), head
  const int32_t* block_table;
  int bt_stride;
  const int32_t* cache_batch_idx;
  const int32_t* seqlens;
  int32_t* seqlens_out;
  int B, Snew, Hq, Hkv, D, page_size, num_pages;
  const float *cos, *sin;
  int rot_dim, rot_positions, interleaved;
  int q_rows;  // B * Snew * Hq when q is given, else 0
  int* status;
};

__device__ __forceinline__ void unpack8(uint4 u, float* f) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}
__device__ __forceinline__ uint4 pack8(const float* f) {
  uint4 u;
  uint32_t* w = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    w[i] = *reinterpret_cast<const uint32_t*>(&h);
  }
  return u;
}

// Rotates chunk c (elements 8c .. 8c+7) of the row at `src` (row base) by the
// angles of position pos; returns the chunk's 8 results in out.
__device__ __forceinline__ void rotate_chunk(const KvUpdateArgs& a, const __nv_bfloat16* src, int c, int pos,
                                             float* out) {
  float x[8];
  unpack8(*reinterpret_cast<const uint4*>(src + 8 * c), x);
  const int e0 = 8 * c;
  if (a.cos == nullptr || e0 >= a.rot_dim) {
#pragma unroll
    for (int e = 0; e < 8; ++e) out[e] = x[e];
    return;
  }
  const float* cs = a.cos + (int64_t)pos * (a.rot_dim / 2);
  const float* sn = a.sin + (int64_t)pos * (a.rot_dim / 2);
  if (a.interleaved) {
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const int j = e0 / 2 + p;
      const float c0 = cs[j], s0 = sn[j];
      out[2 * p] = x[2 * p] * c0 - x[2 * p + 1] * s0;
      out[2 * p + 1] = x[2 * p] * s0 + x[2 * p + 1] * c0;
    }
  } else {
    const int half = a.rot_dim / 2;
    const bool first = e0 < half;
    float y[8];  // the partner chunk
    unpack8(*reinterpret_cast<const uint4*>(src + (first ? e0 + half : e0 - half)), y);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int j = first ? e0 + e : e0 + e - half;
      const float c0 = cs[j], s0 = sn[j];
      out[e] = first ? x[e] * c0 - y[e] * s0 : y[e] * s0 + x[e] * c0;
    }
  }
}

__global__ void __launch_bounds__(256) kvcache_update_kernel(const KvUpdateArgs a) {
  const int chunks = a.D / 8;
  const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t kv_rows = a.k_new ? (int64_t)a.B * a.Snew * a.Hkv : 0;
  const int64_t row = tid / chunks;
  const int c = (int)(tid % chunks);
  if (a.seqlens_out && tid < a.B) a.seqlens_out[tid] = a.seqlens[tid] + a.Snew;
  if (row >= a.q_rows + kv_rows) return;
  const bool is_q = row < a.q_rows;
  const int64_t r = is_q ? row : row - a.q_rows;
  const int H = is_q ? a.Hq : a.Hkv;
  const int h = (int)(r % H);
  const int i = (int)((r / H) % a.Snew);
  const int b = (int)(r / ((int64_t)H * a.Snew));
  const int pos = a.seqlens[b] + i;
  if (pos < 0 || (a.cos != nullptr && pos >= a.rot_positions)) {
    if (a.status && c == 0) atomicOr(a.status, KV_BAD_LEN);
    return;
  }
  float out[8];
  if (is_q) {
    rotate_chunk(a, a.q + b * a.q_sb + (int64_t)i * a.q_ss + (int64_t)h * a.q_sh, c, pos, out);
    *reinterpret_cast<uint4*>(a.q_out + b * a.qo_sb + (int64_t)i * a.qo_ss + (int64_t)h * a.qo_sh + 8 * c) =
        pack8(out);
    return;
  }
  // cache row of position pos
  int64_t page;
  int slot;
  if (a.block_table) {
    const int lp = pos / a.page_size;
    slot = pos % a.page_size;
    if (lp >= a.bt_stride) {
      if (a.status && c == 0) atomicOr(a.status, KV_BAD_PAGE);
      return;
    }
    page = a.block_table[(int64_t)b * a.bt_stride + lp];
  } else {
    page = a.cache_batch_idx ? a.cache_batch_idx[b] : b;
    slot = pos;
    if (pos >= a.page_size) {
      if (a.status && c == 0) atomicOr(a.status, KV_BAD_LEN);
      return;
    }
  }
  if (page < 0 || page >= a.num_pages) {
    if (a.status && c == 0) atomicOr(a.status, KV_BAD_PAGE);
    return;
  }
  const int64_t dst = page * a.c_sp + (int64_t)slot * a.c_ss + (int64_t)h * a.c_sh + 8 * c;
  rotate_chunk(a, a.k_new + b * a.kn_sb + (int64_t)i * a.kn_ss + (int64_t)h * a.kn_sh, c, pos, out);
  *reinterpret_cast<uint4*>(a.k_cache + dst) = pack8(out);
  *reinterpret_cast<uint4*>(a.v_cache + dst) =
      *reinterpret_cast<const uint4*>(a.v_new + b * a.vn_sb + (int64_t)i * a.vn_ss + (int64_t)h * a.vn_sh + 8 * c);
}

}  // namespace attn_kv_kernels
