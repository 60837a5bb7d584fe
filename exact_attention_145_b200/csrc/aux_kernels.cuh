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
  int64_t doc_bstride;  // elements between the document rows of batches; 0 = one shared row
  int Bm, Hm;           // batch and head slices of the tables: [Bm][Hm][nQ][nK]
  int Sq, Skv, blk_q, blk_kv, nQ, nK;
  uint8_t* cls;
  int32_t *part_cnt, *part_idx, *full_cnt, *full_idx;
  int32_t* row_order;   // [Bm][nQ]
  int32_t* doc_start;   // [Bm][Sq] (document masks)
  int32_t* doc_sorted;  // [Bm]     (document masks)
};

// Block-mask build, pass 1: classify tiles (0 empty, 1 partial, 2 full).
// Only in-range positions of ragged edge tiles count.
constexpr int kMaskThreads = 128;
constexpr int kKvPerCta = 8;
constexpr int kRunPerThread = 8;  // ids per thread per shared-memory segment of doc_runs_kernel

// Window forms (none, causal, window): one thread per tile, exact interval
// arithmetic. The keys a query at position p may see form the window
// [p - wl, p + wr] (a side with a negative bound is unbounded). Over a tile's
// rows q0..q1 these windows overlap or touch, so their union is the single
// interval [q0 - wl, q1 + wr]: the tile is empty iff its keys k0..k1 miss that
// interval, and full iff every key lies in every row's window,
// i.e. k0 >= q1 - wl and k1 <= q0 + wr.
__global__ void __launch_bounds__(256) classify_range_kernel(const MaskArgs a) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (int64_t)a.nQ * a.nK) return;
  const int qt = (int)(i / a.nK), kt = (int)(i % a.nK);
  const long q0 = (long)qt * a.blk_q + a.q_offset;
  const long q1 = (long)min((qt + 1) * a.blk_q, a.Sq) - 1 + a.q_offset;
  const long k0 = (long)kt * a.blk_kv;
  const long k1 = (long)min((kt + 1) * a.blk_kv, a.Skv) - 1;
  bool empty = false, full = true;
  if (a.kind != 0) {
    if (a.wl >= 0) {
      if (k1 < q0 - a.wl) empty = true;
      if (k0 < q1 - a.wl) full = false;
    }
    if (a.wr >= 0) {
      if (k0 > q1 + a.wr) empty = true;
      if (k1 > q0 + a.wr) full = false;
    }
  }
  a.cls[i] = empty ? 0 : (full ? 2 : 1);
}

__device__ __forceinline__ void warp_minmax(int& lo, int& hi) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, off));
    hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, off));
  }
}

// Document mask (key j visible to query i iff doc[j] == doc[i] and j <= i):
// one CTA per (q-tile, kKvPerCta kv-tiles). The id ranges of the two sides
// decide most tiles at once: keys all past the last query -> empty; disjoint
// id ranges -> empty; one id shared by every position of both tiles -> the
// causal class. The remaining tiles (those crossing a document boundary, or
// any tile when the ids are not grouped) are evaluated pair by pair: each
// thread walks its query rows against the tile's keys, stopping once it has
// seen both an allowed and a masked pair, and block votes give "any" and "all".
// Batch slice b = blockIdx.z reads document row b and writes head slice 0 of
// batch slice b.
__global__ void __launch_bounds__(kMaskThreads) classify_doc_kernel(MaskArgs a) {
  extern __shared__ int doc_k[];  // [kKvPerCta * blk_kv] key doc ids
  __shared__ int red_lo[kMaskThreads / 32], red_hi[kMaskThreads / 32];
  __shared__ int tile_lo[kKvPerCta], tile_hi[kKvPerCta];
  a.doc_id += (int64_t)blockIdx.z * a.doc_bstride;
  a.cls += (int64_t)blockIdx.z * a.Hm * a.nQ * a.nK;
  const int qt = blockIdx.x;
  const int kt0 = blockIdx.y * kKvPerCta;
  const int kt1 = min(kt0 + kKvPerCta, a.nK);
  const int q0 = qt * a.blk_q;
  const int rows = min(a.blk_q, a.Sq - q0);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int k_first = kt0 * a.blk_kv, k_end = min(kt1 * a.blk_kv, a.Skv);
  if (k_first > q0 + rows - 1) {
    // every key of these tiles lies past the last query of the row tile:
    // all empty under the causal document mask, no ids needed
    // (head slice 0, like the classification below; the compaction copies it)
    for (int kt = kt0 + threadIdx.x; kt < kt1; kt += blockDim.x) a.cls[(int64_t)qt * a.nK + kt] = 0;
    return;
  }
  for (int c = threadIdx.x; c < k_end - k_first; c += blockDim.x) doc_k[c] = a.doc_id[k_first + c];
  // id range of the query tile
  int lo = 0x7fffffff, hi = -0x7fffffff - 1;
  for (int r = threadIdx.x; r < rows; r += blockDim.x) {
    const int d = a.doc_id[q0 + r];
    lo = min(lo, d);
    hi = max(hi, d);
  }
  warp_minmax(lo, hi);
  if (lane == 0) {
    red_lo[warp] = lo;
    red_hi[warp] = hi;
  }
  __syncthreads();
  int qlo = red_lo[0], qhi = red_hi[0];
#pragma unroll
  for (int w = 1; w < kMaskThreads / 32; ++w) {
    qlo = min(qlo, red_lo[w]);
    qhi = max(qhi, red_hi[w]);
  }
  // id range of each key tile, one warp per tile
  for (int kt = kt0 + warp; kt < kt1; kt += kMaskThreads / 32) {
    const int base = (kt - kt0) * a.blk_kv;
    const int cols = min(a.blk_kv, a.Skv - kt * a.blk_kv);
    int l2 = 0x7fffffff, h2 = -0x7fffffff - 1;
    for (int c = lane; c < cols; c += 32) {
      l2 = min(l2, doc_k[base + c]);
      h2 = max(h2, doc_k[base + c]);
    }
    warp_minmax(l2, h2);
    if (lane == 0) {
      tile_lo[kt - kt0] = l2;
      tile_hi[kt - kt0] = h2;
    }
  }
  __syncthreads();
  for (int kt = kt0; kt < kt1; ++kt) {
    const int k0 = kt * a.blk_kv;
    const int cols = min(a.blk_kv, a.Skv - k0);
    const int klo = tile_lo[kt - kt0], khi = tile_hi[kt - kt0];
    int cls;
    if (k0 > q0 + rows - 1 || khi < qlo || klo > qhi) {
      cls = 0;
    } else if (qlo == qhi && klo == khi && qlo == klo) {
      cls = (k0 + cols - 1 <= q0) ? 2 : 1;
    } else {
      // Eight keys per iteration from two 16-byte shared loads (blk_kv is a
      // multiple of 16, so every group starts 32-byte aligned); keys past
      // the ragged end of the sequence are skipped.
      const int4* dk4 = reinterpret_cast<const int4*>(doc_k + (kt - kt0) * a.blk_kv);
      bool any = false, all = true;
      for (int r = threadIdx.x; r < rows && (all || !any); r += blockDim.x) {
        const int qi = q0 + r;
        const int di = a.doc_id[qi];
        for (int c = 0; c < cols && (all || !any); c += 8) {
          const int4 d0 = dk4[c / 4], d1 = dk4[c / 4 + 1];
          const int dd[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            if (c + e < cols) {
              const bool ok = k0 + c + e <= qi && dd[e] == di;
              any |= ok;
              all &= ok;
            }
          }
        }
      }
      const int any_b = __syncthreads_or(any);
      const int all_b = __syncthreads_and(all);
      cls = any_b ? (all_b ? 2 : 1) : 0;
    }
    if (threadIdx.x == 0) a.cls[(int64_t)qt * a.nK + kt] = (uint8_t)cls;
  }
}

// Pass 2: one warp per (slice, q-tile) compacts the class row into the
// ascending partial and full lists with ballots. Pass 1 classified head slice
// 0 of the first b_class batch slices; every other slice copies its class row
// from head slice 0 of batch slice (b < b_class ? b : 0) first.
__global__ void __launch_bounds__(32) compact_lists_kernel(const MaskArgs a, int b_class) {
  const int qt = blockIdx.x;
  const int slice = blockIdx.y;  // b * Hm + h
  const int b = slice / a.Hm;
  const int lane = threadIdx.x;
  const int64_t tiles = (int64_t)a.nQ * a.nK;
  uint8_t* row = a.cls + slice * tiles + (int64_t)qt * a.nK;
  const uint8_t* src = a.cls + (int64_t)(b < b_class ? b : 0) * a.Hm * tiles + (int64_t)qt * a.nK;
  const bool copy = src != row;
  int32_t* pidx = a.part_idx + slice * tiles + (int64_t)qt * a.nK;
  int32_t* fidx = a.full_idx + slice * tiles + (int64_t)qt * a.nK;
  int np = 0, nf = 0;
  for (int k0 = 0; k0 < a.nK; k0 += 32) {
    const int kt = k0 + lane;
    const uint8_t c = kt < a.nK ? src[kt] : 0;
    if (copy && kt < a.nK) row[kt] = c;
    const unsigned mp = __ballot_sync(0xffffffffu, c == 1);
    const unsigned mf = __ballot_sync(0xffffffffu, c == 2);
    const unsigned below = (1u << lane) - 1u;
    if (c == 1) pidx[np + __popc(mp & below)] = kt;
    if (c == 2) fidx[nf + __popc(mf & below)] = kt;
    np += __popc(mp);
    nf += __popc(mf);
  }
  if (lane == 0) {
    a.part_cnt[(int64_t)slice * a.nQ + qt] = np;
    a.full_cnt[(int64_t)slice * a.nQ + qt] = nf;
  }
}

// Pass 3: the work order of batch slice b = blockIdx.x: its q-tiles by
// decreasing number of visited kv tiles (head slice 0), ties by index, so the
// persistent attention kernel hands out the longest rows first. Each thread
// ranks its q-tiles by counting the tiles that come before them.
constexpr int kOrderThreads = 256;
__global__ void __launch_bounds__(kOrderThreads) row_order_kernel(const MaskArgs a) {
  const int b = blockIdx.x;
  const int64_t base = (int64_t)b * a.Hm * a.nQ;  // head slice 0 of batch slice b
  for (int i = threadIdx.x; i < a.nQ; i += blockDim.x) {
    const int wi = a.part_cnt[base + i] + a.full_cnt[base + i];
    int rank = 0;
    for (int j = 0; j < a.nQ; ++j) {
      const int wj = a.part_cnt[base + j] + a.full_cnt[base + j];
      rank += (wj > wi) || (wj == wi && j < i);
    }
    a.row_order[(int64_t)b * a.nQ + rank] = i;
  }
}

// Document masks, batch slice b = blockIdx.x (document row b, or row 0 when
// the rows are shared): doc_start[i] = first position of the run of equal
// ids that holds i, and doc_sorted = 1 when the ids never decrease (then
// every document is a single run and key j <= i is allowed iff
// j >= doc_start[i]). Each thread scans a contiguous chunk; the chunks'
// last run starts are combined with a block-wide max scan.
constexpr int kRunThreads = 1024;
__global__ void __launch_bounds__(kRunThreads) doc_runs_kernel(const MaskArgs a) {
  // The ids are staged segment by segment in shared memory with coalesced
  // loads (each thread then scans kRunPerThread consecutive ids there), and
  // the run starts go back through the same buffer with coalesced stores.
  __shared__ int seg[kRunThreads * kRunPerThread];
  __shared__ int warp_max[kRunThreads / 32];
  const int b = blockIdx.x;
  const int32_t* doc = a.doc_id + (int64_t)b * a.doc_bstride;
  int32_t* out = a.doc_start + (int64_t)b * a.Sq;
  const int S = a.Sq;
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
  constexpr int kSeg = kRunThreads * kRunPerThread;
  int carry = -1;        // last run start before the segment
  int prev_id = 0;       // id just before the segment (valid when seg0 > 0)
  bool decreasing = false;
  for (int seg0 = 0; seg0 < S; seg0 += kSeg) {
    const int n = min(kSeg, S - seg0);
    for (int c = threadIdx.x; c < n; c += kRunThreads) seg[c] = doc[seg0 + c];
    __syncthreads();
    const int i0 = min(n, (int)threadIdx.x * kRunPerThread), i1 = min(n, i0 + kRunPerThread);
    // ids read before any thread rewrites the buffer: the one before this
    // thread's range, and the segment's last
    const int first_prev = i0 > 0 ? seg[i0 - 1] : prev_id;
    const int last_id = seg[n - 1];
    int last = -1;
    for (int i = i0; i < i1; ++i) {
      const int d = seg[i];
      const int dp = i > 0 ? seg[i - 1] : prev_id;
      const bool start = (seg0 + i == 0) || d != dp;
      if (start) last = seg0 + i;
      if (seg0 + i > 0 && d < dp) decreasing = true;
    }
    // inclusive max scan of `last` over threads: warps, then the warp totals
    int incl = last;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl = max(incl, v);
    }
    if (lane == 31) warp_max[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      int w = warp_max[lane];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, w, off);
        if (lane >= off) w = max(w, v);
      }
      warp_max[lane] = w;  // inclusive over warps 0..lane
    }
    __syncthreads();
    const int before_warp = warp > 0 ? warp_max[warp - 1] : -1;
    const int excl_lane = __shfl_up_sync(0xffffffffu, incl, 1);
    int cur = max(carry, max(before_warp, lane > 0 ? excl_lane : -1));
    const int seg_last = warp_max[kRunThreads / 32 - 1];
    // run starts in place of the ids (each thread reads and rewrites only its
    // own range; the id before it was saved above)
    int dp = first_prev;
    for (int i = i0; i < i1; ++i) {
      const int d = seg[i];
      if ((seg0 + i == 0) || d != dp) cur = seg0 + i;
      dp = d;
      seg[i] = cur;
    }
    __syncthreads();
    for (int c = threadIdx.x; c < n; c += kRunThreads) out[seg0 + c] = seg[c];
    carry = max(carry, seg_last);
    prev_id = last_id;
    __syncthreads();
  }
  const int any_dec = __syncthreads_or(decreasing ? 1 : 0);
  if (threadIdx.x == 0) a.doc_sorted[b] = any_dec ? 0 : 1;
}

// One warp per output row: lse = ln sum_i exp(lse_i); o = sum_i exp(lse_i - lse) o_i.
struct CombineArgs {
  const float* o_parts;    // [rows][n][D]
  const float* lse_parts;  // [rows][n]
  int rows, n, D;
  int rows_per_b;          // rows are (b, r) with r < rows_per_b, r = token * heads + h
  int heads;
  __nv_bfloat16* o;
  int64_t o_sb, o_st, o_sh;  // element strides of the output rows (b, token, h)
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
  const int b = row / a.rows_per_b, r = row % a.rows_per_b;
  const int tok = r / a.heads, h = r % a.heads;
  __nv_bfloat16* dst = a.o + (int64_t)b * a.o_sb + (int64_t)tok * a.o_st + (int64_t)h * a.o_sh + lane * V;
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
