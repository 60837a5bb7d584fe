// fwd_kernel.cuh - the attention forward kernel for sm_100a, shared by the
// prefill path (attn_fwd) and the split-KV paged decode path (attn_decode).
//
// One CTA owns two 128-row query sub-tiles ("subtiles" 0 and 1) and streams
// 128-key K/V tiles through shared memory. Warp roles (320 threads):
//   warps 0-3  softmax for subtile 0 (thread t owns query row t = TMEM lane t)
//   warps 4-7  softmax for subtile 1
//   warp  8    tcgen05 MMA issue (one elected lane); owns the TMEM allocation
//   warp  9    TMA producer (one elected lane)
// The tensor pipe alternates between the subtiles so that one subtile's
// softmax overlaps the other's MMAs: on B200 the exponentials take about
// twice as long as the two GEMMs of a tile, so a single query tile per CTA
// would leave the tensor cores idle ("FlexAttention + FlashAttention-4" talk,
// the two-Q-tile ping-pong pipeline). MMA order per step:
//   PV(0, j) QK(0, j+1) PV(1, j) QK(1, j+1)
// TMEM (512 columns): S0 | S1 | O0 | O1. P (bf16) overwrites the first half of
// its S region once the softmax has read S into registers, and feeds the PV
// MMA straight from TMEM. tcgen05.mma ops of one thread execute in issue
// order, so QK(s, j+1) overwrites S(s) only after PV(s, j) has read P(s).
//
// Online softmax ("A Deep Dive into Flash Attention", section "2. Online
// Softmax"), in base 2: x = log2(e) * score; each row keeps a reference max
// m and a running sum l; O is rescaled by 2^(m_old - m_new) only when some
// row of the warp sees its max grow by more than 8 (probabilities stay below
// 2^8, which bf16 P and the fp32 accumulators absorb exactly as well).
// Because QK(s, j+1) is committed after PV(s, j), seeing S(s, j+1) ready
// implies O(s) is settled, so the rescale needs no extra wait.
//
// Prefill pairs the subtiles either as two query heads of one KV group over
// the same 128 rows (GQA, group size even: identical masks, K/V shared) or as
// two consecutive 128-row tiles of one head (MHA). Decode puts all query
// heads of a KV group on the 128 MMA rows and gives the two subtiles
// alternating key tiles of the split; their partial results are merged in
// the CTA before one partial (O_i, LSE_i) per split is written.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "sm100.cuh"

namespace attn_kernels {

using namespace attn_sm100;

constexpr int kRows = 128;      // query rows per subtile (MMA M)
constexpr int kKeys = 128;      // keys per K/V tile (MMA N of QK^T, K of PV)
constexpr int kThreads = 320;
constexpr int kMmaWarp = 8;
constexpr int kTmaWarp = 9;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

enum : int { MASK_NONE = 0, MASK_CAUSAL = 1, MASK_WINDOW = 2, MASK_DOCUMENT = 3 };
enum : int { MOD_NONE = 0, MOD_SOFTCAP = 1, MOD_ALIBI = 2 };
enum : int { DEV_TIMEOUT = 1, DEV_BAD_PAGE = 2 };

struct FwdArgs {
  int B, Hq, Hkv, Sq, Skv, g;
  float scale_log2;     // softmax scale * log2(e)
  float scale;          // softmax scale
  int mask, wl, wr, q_offset;
  const int32_t* doc_id;
  const uint8_t* bm_cls;  // [nQ][nK] class table or nullptr
  int nQ, nK;
  int mod;
  float softcap;
  const float* alibi;
  int alibi_bstride;
  // prefill outputs
  __nv_bfloat16* o;
  int64_t o_sb, o_ss, o_sh;
  float* lse;
  int pair_heads;  // 1: subtiles are heads (2u, 2u+1) over one row tile; 0: consecutive row tiles
  int n_row_units; // prefill: number of row-tile units per (b, head unit)
  // decode
  const int32_t* block_table;
  int bt_stride;
  const int32_t* seqlens;
  int page_size, num_pages, box_rows, n_splits, tiles_per_split;
  float* part_o;    // [B][Hq][n_splits][D]
  float* part_lse;  // [B][Hq][n_splits]
  int* status;
};

template <int D, bool DECODE>
struct Layout {
  static constexpr int kNSlot = DECODE ? (D == 128 ? 3 : 6) : (D == 128 ? 2 : 5);
  static constexpr int kNQ = DECODE ? 1 : 2;
  static constexpr int kTileBytes = kKeys * D * 2;  // one K or V tile (== one Q subtile)
  static constexpr int kChunk = 128 * 64 * 2;       // one 128-row x 64-col SW128 box
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + kNQ * kTileBytes;
  static constexpr int kVOff = kKOff + kNSlot * kTileBytes;
  static constexpr int kBarOff = kVOff + kNSlot * kTileBytes;
  static constexpr int kSmemBytes = kBarOff + 1024 + 2 * 128 * 4 + 1024;  // + barriers + merge scratch + align slack
  static constexpr int kOCols = D;  // TMEM columns of one O accumulator
};

struct Barriers {
  uint64_t q_full;
  uint64_t k_full[6];
  uint64_t v_full[6];
  uint64_t kv_empty[6];
  uint64_t s_ready[2];
  uint64_t p_ready[2];
  uint64_t o_done[2];
  uint64_t final_mma;
  uint32_t tmem_base;
  int abort_flag;
};

// ---------------------------------------------------------------- work map
struct Work {
  int b, hk;
  int head[2];  // query head of each subtile (prefill) / first head of the group (decode)
  int row0[2];  // first query row of each subtile (prefill)
  int split;    // decode
  int t_begin, t_end;  // decode: key tiles [t_begin, t_end) of this split
  int seqlen;          // decode
};

template <bool DECODE>
__device__ __forceinline__ Work map_work(const FwdArgs& a) {
  Work w;
  const int u = blockIdx.x;
  if constexpr (DECODE) {
    w.split = u % a.n_splits;
    const int bh = u / a.n_splits;
    w.hk = bh % a.Hkv;
    w.b = bh / a.Hkv;
    w.head[0] = w.head[1] = w.hk * a.g;
    w.row0[0] = w.row0[1] = 0;
    w.seqlen = a.seqlens[w.b];
    const int nt = (max(w.seqlen, 0) + kKeys - 1) / kKeys;
    w.t_begin = min(nt, w.split * a.tiles_per_split);
    w.t_end = min(nt, w.t_begin + a.tiles_per_split);
  } else {
    // Heaviest row tiles first: unit index u walks row tiles from the end.
    const int HU = a.pair_heads ? a.Hq / 2 : a.Hq;
    const int per = a.B * HU;
    const int qi = u / per, rem = u % per;
    w.b = rem / HU;
    const int hu = rem % HU;
    const int rt = a.n_row_units - 1 - qi;
    if (a.pair_heads) {
      w.head[0] = 2 * hu;
      w.head[1] = 2 * hu + 1;
      w.row0[0] = w.row0[1] = rt * kRows;
    } else {
      w.head[0] = w.head[1] = hu;
      w.row0[0] = 2 * rt * kRows;
      w.row0[1] = w.row0[0] + kRows;
    }
    w.hk = w.head[0] / a.g;
    w.split = 0;
    w.t_begin = w.t_end = 0;
    w.seqlen = 0;
  }
  return w;
}

// Tile class of kv tile t for subtile s: 0 empty, 1 partial, 2 full.
template <bool DECODE>
__device__ __forceinline__ int tile_class(const FwdArgs& a, const Work& w, int s, int t) {
  if constexpr (DECODE) {
    (void)s;
    if (t < w.t_begin || t >= w.t_end) return 0;
    return (t + 1) * kKeys <= w.seqlen ? 2 : 1;
  } else {
    const int r0 = w.row0[s];
    if (r0 >= a.Sq || t >= a.nK) return 0;
    const int r1 = min(r0 + kRows, a.Sq) - 1;
    const int c0 = t * kKeys;
    const int c1 = min(c0 + kKeys, a.Skv) - 1;
    const bool ragged = c0 + kKeys > a.Skv;
    int cls;
    if (a.bm_cls != nullptr) {
      cls = a.bm_cls[(r0 / kRows) * a.nK + t];
    } else if (a.mask == MASK_NONE) {
      cls = 2;
    } else {
      // window form: q_pos - left <= kv <= q_pos + right (causal: left = -1, right = 0)
      const long p0 = (long)r0 + a.q_offset, p1 = (long)r1 + a.q_offset;
      bool empty = false, full = true;
      if (a.wl >= 0) {
        if ((long)c1 < p0 - a.wl) empty = true;
        if ((long)c0 < p1 - a.wl) full = false;
      }
      if (a.wr >= 0) {
        if ((long)c0 > p1 + a.wr) empty = true;
        if ((long)c1 > p0 + a.wr) full = false;
      }
      cls = empty ? 0 : (full ? 2 : 1);
    }
    if (ragged && cls == 2) cls = 1;
    return cls;
  }
}

// Step sequence: prefill step i uses the i-th kv tile with a non-empty class
// for either subtile; decode step i gives subtile s the tile t_begin + 2i + s.
template <bool DECODE>
__device__ __forceinline__ int num_steps(const FwdArgs& a, const Work& w) {
  if constexpr (DECODE) {
    return (w.t_end - w.t_begin + 1) / 2;
  } else {
    int n = 0;
    for (int t = 0; t < a.nK; ++t)
      if (tile_class<false>(a, w, 0, t) | tile_class<false>(a, w, 1, t)) ++n;
    return n;
  }
}

// Advances a prefill tile cursor to the next tile any subtile needs.
__device__ __forceinline__ int next_tile(const FwdArgs& a, const Work& w, int t) {
  ++t;
  while (t < a.nK && (tile_class<false>(a, w, 0, t) | tile_class<false>(a, w, 1, t)) == 0) ++t;
  return t;
}

// ---------------------------------------------------------------- producer
template <int D, bool DECODE>
__device__ __forceinline__ void load_kv_tile(const FwdArgs& a, const Work& w, const CUtensorMap* mk,
                                             const CUtensorMap* mv, uint8_t* kdst, uint8_t* vdst, uint64_t* kbar,
                                             uint64_t* vbar, int t, bool absent) {
  using L = Layout<D, DECODE>;
  mbar_arrive_expect_tx(kbar, L::kTileBytes);
  mbar_arrive_expect_tx(vbar, L::kTileBytes);
  if constexpr (DECODE) {
    const int rows = a.box_rows;
    for (int u = 0; u < kKeys / rows; ++u) {
      const int tok = t * kKeys + u * rows;
      const int lp = tok / a.page_size;
      const int slot = tok % a.page_size;
      int phys = a.num_pages;  // out of range -> TMA fills zeros, no memory read
      if (!absent && tok < w.seqlen && lp < a.bt_stride) {
        const int pg = a.block_table[(int64_t)w.b * a.bt_stride + lp];
        if (pg >= 0 && pg < a.num_pages) {
          phys = pg;
        } else if (a.status) {
          atomicOr(a.status, DEV_BAD_PAGE);
        }
      }
      for (int c = 0; c < D / 64; ++c) {
        tma_load_4d(kdst + c * L::kChunk + u * rows * 128, mk, kbar, c * 64, w.hk, slot, phys);
        tma_load_4d(vdst + c * L::kChunk + u * rows * 128, mv, vbar, c * 64, w.hk, slot, phys);
      }
    }
  } else {
    (void)absent;
    for (int c = 0; c < D / 64; ++c) {
      tma_load_4d(kdst + c * L::kChunk, mk, kbar, c * 64, t * kKeys, w.hk, w.b);
      tma_load_4d(vdst + c * L::kChunk, mv, vbar, c * 64, t * kKeys, w.hk, w.b);
    }
  }
}

// ---------------------------------------------------------------- softmax
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcp(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Per-row state of one query row.
struct RowState {
  float m;  // reference max (log2 units), -inf until a key is seen
  float l;  // running sum of 2^(x - m)
};

template <int D, bool DECODE>
__device__ __forceinline__ void softmax_step(const FwdArgs& a, const Work& w, int s, int row, int t, int cls,
                                             uint32_t tS, uint32_t tO, bool first, RowState& st) {
  float x[kKeys];
  const float NEG_INF = -__int_as_float(0x7f800000);
  if (cls == 0) {
#pragma unroll
    for (int c = 0; c < kKeys; ++c) x[c] = NEG_INF;
  } else {
    tmem_ld32f(tS + 0, x);
    tmem_ld32f(tS + 32, x + 32);
    tmem_ld32f(tS + 64, x + 64);
    tmem_ld32f(tS + 96, x + 96);
    tmem_ld_wait();
    reg_fence_f<kKeys>(x);
    // Score mods on the scaled score, expressed in log2 units.
    const int qrow = DECODE ? 0 : w.row0[s] + row;
    const long q_pos = DECODE ? (long)w.seqlen - 1 : (long)qrow + a.q_offset;
    const int head = w.head[s] + (DECODE ? row : 0);
    if (a.mod == MOD_NONE) {
#pragma unroll
      for (int c = 0; c < kKeys; ++c) x[c] *= a.scale_log2;
    } else if (a.mod == MOD_SOFTCAP) {
      // c * tanh(y), y = s / c, with tanh(y) = 1 - 2 / (e^{2y} + 1)
      const float k2 = 2.0f * a.scale / a.softcap * kLog2e;
      const float cl = a.softcap * kLog2e;
#pragma unroll
      for (int c = 0; c < kKeys; ++c) {
        const float e = ex2(x[c] * k2);
        x[c] = cl * (1.0f - 2.0f * rcp(e + 1.0f));
      }
    } else {
      const float slope = a.alibi[(int64_t)w.b * a.alibi_bstride + min(head, a.Hq - 1)] * kLog2e;
      const float base = slope * (float)((long)t * kKeys - q_pos);
#pragma unroll
      for (int c = 0; c < kKeys; ++c) x[c] = fmaf(x[c], a.scale_log2, fmaf(slope, (float)c, base));
    }
    if (cls == 1) {
      const int kv0 = t * kKeys;
      if constexpr (DECODE) {
#pragma unroll
        for (int c = 0; c < kKeys; ++c)
          if (kv0 + c >= w.seqlen) x[c] = NEG_INF;
      } else {
        const int Skv = a.Skv;
        if (a.mask == MASK_DOCUMENT) {
          const int dq = a.doc_id[min(qrow, a.Sq - 1)];
#pragma unroll
          for (int c = 0; c < kKeys; ++c) {
            const int kv = kv0 + c;
            const bool ok = kv < Skv && (long)kv <= q_pos && __ldg(a.doc_id + min(kv, Skv - 1)) == dq;
            if (!ok) x[c] = NEG_INF;
          }
        } else {
          const long lo = a.wl >= 0 ? q_pos - a.wl : -(1l << 40);
          const long hi = a.wr >= 0 ? q_pos + a.wr : (1l << 40);
#pragma unroll
          for (int c = 0; c < kKeys; ++c) {
            const int kv = kv0 + c;
            const bool ok = kv < Skv && (long)kv >= lo && (long)kv <= hi;
            if (!ok) x[c] = NEG_INF;
          }
        }
      }
    }
  }
  // Row max over the tile.
  float m0 = x[0], m1 = x[1], m2 = x[2], m3 = x[3];
#pragma unroll
  for (int c = 4; c < kKeys; c += 4) {
    m0 = fmaxf(m0, x[c]);
    m1 = fmaxf(m1, x[c + 1]);
    m2 = fmaxf(m2, x[c + 2]);
    m3 = fmaxf(m3, x[c + 3]);
  }
  const float mt = fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
  const bool grow = mt > st.m + kRescaleThreshold;  // true whenever st.m == -inf and mt is finite
  const bool warp_rescale = __any_sync(0xffffffffu, grow);
  float alpha = 1.0f;
  if (warp_rescale) {
    const float m_new = fmaxf(st.m, mt);
    alpha = (m_new == NEG_INF) ? 1.0f : ex2(st.m - m_new);
    st.l *= alpha;
    st.m = m_new;
  }
  const float mu = (st.m == NEG_INF) ? 0.0f : st.m;
  float l0 = 0.f, l1 = 0.f;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t pk[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const float p0 = ex2(x[64 * h + 2 * j] - mu);
      const float p1 = ex2(x[64 * h + 2 * j + 1] - mu);
      l0 += p0;
      l1 += p1;
      pk[j] = pack_bf16x2(p0, p1);
    }
    tmem_st32(tS + 32 * h, pk);
  }
  st.l += l0 + l1;
  if (warp_rescale && !first) {
    // O(s) is settled: PV(s, step-1) completed before S(s, step) was
    // committed, and PV(s, step) is issued only after this thread arrives.
#pragma unroll
    for (int c = 0; c < D; c += 32) {
      float o[32];
      tmem_ld32f(tO + c, o);
      tmem_ld_wait();
      reg_fence_f<32>(o);
      uint32_t ob[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) ob[j] = __float_as_uint(o[j] * alpha);
      tmem_st32(tO + c, ob);
    }
  }
  tmem_st_wait();
}

// ---------------------------------------------------------------- kernel
template <int D, bool DECODE>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                    const __grid_constant__ CUtensorMap map_v, const FwdArgs a) {
  using L = Layout<D, DECODE>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Barriers& bar = *reinterpret_cast<Barriers*>(smem + L::kBarOff);
  float* merge_m = reinterpret_cast<float*>(smem + L::kBarOff + 1024);
  float* merge_l = merge_m + 128;
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  volatile int* abort_flag = &bar.abort_flag;

  const Work w = map_work<DECODE>(a);
  const int n = num_steps<DECODE>(a, w);

  if (threadIdx.x == 0) {
    bar.abort_flag = 0;
    mbar_init(&bar.q_full, 1);
    for (int i = 0; i < L::kNSlot; ++i) {
      mbar_init(&bar.k_full[i], 1);
      mbar_init(&bar.v_full[i], 1);
      mbar_init(&bar.kv_empty[i], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar.s_ready[s], 1);
      mbar_init(&bar.p_ready[s], 128);
      mbar_init(&bar.o_done[s], 1);
    }
    mbar_init(&bar.final_mma, 1);
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&bar.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar.tmem_base;

  if (warp == kTmaWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && n > 0) {
      tma_prefetch_desc(&map_q);
      tma_prefetch_desc(&map_k);
      tma_prefetch_desc(&map_v);
      mbar_arrive_expect_tx(&bar.q_full, L::kNQ * L::kTileBytes);
      for (int s = 0; s < L::kNQ; ++s)
        for (int c = 0; c < D / 64; ++c) {
          uint8_t* dst = smem + L::kQOff + s * L::kTileBytes + c * L::kChunk;
          if constexpr (DECODE)
            tma_load_3d(dst, &map_q, &bar.q_full, c * 64, w.head[0], w.b);
          else
            tma_load_4d(dst, &map_q, &bar.q_full, c * 64, w.row0[s], w.head[s], w.b);
        }
      const int n_loads = DECODE ? 2 * n : n;
      int t = DECODE ? w.t_begin : next_tile(a, w, -1);
      int issued = 0;
      for (int k = 0; k < n_loads; ++k) {
        const int slot = k % L::kNSlot;
        const int use = k / L::kNSlot;
        if (use > 0 && !mbar_wait(&bar.kv_empty[slot], (use - 1) & 1, abort_flag)) break;
        const bool absent = DECODE && t >= w.t_end;
        load_kv_tile<D, DECODE>(a, w, &map_k, &map_v, smem + L::kKOff + slot * L::kTileBytes,
                                smem + L::kVOff + slot * L::kTileBytes, &bar.k_full[slot], &bar.v_full[slot], t,
                                absent);
        ++issued;
        t = DECODE ? t + 1 : next_tile(a, w, t);
      }
      // Drain: on an abort, wait (bounded) for every copy still in flight so
      // none lands in shared memory after the CTA has exited.
      if (*abort_flag) {
        for (int k = max(0, issued - L::kNSlot); k < issued; ++k) {
          const int slot = k % L::kNSlot;
          const uint32_t par = (k / L::kNSlot) & 1;
          volatile int never = 0;
          mbar_wait(&bar.k_full[slot], par, &never);
          mbar_wait(&bar.v_full[slot], par, &never);
        }
        volatile int never = 0;
        mbar_wait(&bar.q_full, 0, &never);
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0 && n > 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, kKeys, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t q_base = smem_u32(smem + L::kQOff);
      const uint32_t k_base = smem_u32(smem + L::kKOff);
      const uint32_t v_base = smem_u32(smem + L::kVOff);
      auto issue_qk = [&](int s, int slot) {
        const uint32_t qa = q_base + (DECODE ? 0 : s * L::kTileBytes);
        const uint32_t ka = k_base + slot * L::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * L::kChunk + (kk % 4) * 32;
          mma_ss(tmem + s * 128, sdesc_sw128(qa + off, 16, 1024), sdesc_sw128(ka + off, 16, 1024), idesc_qk,
                 kk > 0);
        }
        mma_commit(&bar.s_ready[s]);
      };
      auto issue_pv = [&](int s, int slot, bool acc) {
        const uint32_t va = v_base + slot * L::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < kKeys / 16; ++kk)
          mma_ts(tmem + 256 + s * L::kOCols, tmem + s * 128 + kk * 8, sdesc_sw128(va + kk * 16 * 128, L::kChunk, 1024),
                 idesc_pv, (acc || kk > 0) ? 1u : 0u);
      };
      auto slot_of = [&](int step, int s) { return DECODE ? (2 * step + s) % L::kNSlot : step % L::kNSlot; };
      auto phase_of = [&](int step, int s) {
        return (uint32_t)(((DECODE ? 2 * step + s : step) / L::kNSlot) & 1);
      };
      bool ok = mbar_wait(&bar.q_full, 0, abort_flag);
      tc_fence_after();
      if (ok) ok = mbar_wait(&bar.k_full[slot_of(0, 0)], phase_of(0, 0), abort_flag);
      if (ok) {
        tc_fence_after();
        issue_qk(0, slot_of(0, 0));
        if (DECODE) ok = mbar_wait(&bar.k_full[slot_of(0, 1)], phase_of(0, 1), abort_flag);
        tc_fence_after();
        if (ok) issue_qk(1, slot_of(0, 1));
      }
      for (int j = 0; ok && j < n; ++j) {
        const bool more = j + 1 < n;
#pragma unroll
        for (int s = 0; s < 2; ++s) {
          const int slot = slot_of(j, s);
          if (!mbar_wait(&bar.v_full[slot], phase_of(j, s), abort_flag)) { ok = false; break; }
          if (!mbar_wait(&bar.p_ready[s], j & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          issue_pv(s, slot, j > 0);
          if (!more) mma_commit(&bar.o_done[s]);
          if (DECODE || s == 1) mma_commit(&bar.kv_empty[slot]);
          if (more) {
            const int nslot = slot_of(j + 1, s);
            if (!mbar_wait(&bar.k_full[nslot], phase_of(j + 1, s), abort_flag)) { ok = false; break; }
            tc_fence_after();
            issue_qk(s, nslot);
          }
        }
      }
      // Every MMA must be complete before TMEM is released.
      mma_commit(&bar.final_mma);
      volatile int never = 0;
      mbar_wait(&bar.final_mma, 0, &never);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int s = warp / 4;
    const int row = threadIdx.x % 128;  // TMEM lane
    const uint32_t lane_base = tmem + ((uint32_t)((warp % 4) * 32) << 16);
    const uint32_t tS = lane_base + s * 128;
    const uint32_t tO = lane_base + 256 + s * L::kOCols;
    RowState st;
    st.m = -__int_as_float(0x7f800000);
    st.l = 0.f;
    bool ok = true;
    int t = DECODE ? w.t_begin + s : next_tile(a, w, -1);
    for (int j = 0; j < n; ++j) {
      const int cls = tile_class<DECODE>(a, w, s, t);
      bool got = mbar_wait(&bar.s_ready[s], j & 1, abort_flag);
      got = __all_sync(0xffffffffu, got);
      if (!got) { ok = false; break; }
      tc_fence_after();
      softmax_step<D, DECODE>(a, w, s, row, t, cls, tS, tO, j == 0, st);
      tc_fence_before();
      mbar_arrive(&bar.p_ready[s]);
      t = DECODE ? t + 2 : next_tile(a, w, t);
    }
    // ------------------------------------------------------------ epilogue
    const float NEG_INF = -__int_as_float(0x7f800000);
    if (n > 0 && ok) {
      bool got = mbar_wait(&bar.o_done[s], 0, abort_flag);
      if (DECODE && s == 0) got = got && mbar_wait(&bar.o_done[1], 0, abort_flag);
      got = __all_sync(0xffffffffu, got);
      ok = got;
      tc_fence_after();
    }
    if constexpr (!DECODE) {
      const int qrow = w.row0[s] + row;
      const int h = w.head[s];
      const bool valid = qrow < a.Sq && w.row0[s] < a.Sq;
      const float inv_l = st.l > 0.f ? 1.0f / st.l : 0.f;
      __nv_bfloat16* orow = a.o + (int64_t)w.b * a.o_sb + (int64_t)qrow * a.o_ss + (int64_t)h * a.o_sh;
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        uint32_t o[32];
        if (n > 0 && ok) {
          tmem_ld32(tO + c, o);
          tmem_ld_wait();
          reg_fence(o);
        } else {
#pragma unroll
          for (int j2 = 0; j2 < 32; ++j2) o[j2] = 0u;
        }
        if (valid) {
#pragma unroll
          for (int j2 = 0; j2 < 32; j2 += 8) {
            uint4 v4;
            v4.x = pack_bf16x2(__uint_as_float(o[j2 + 0]) * inv_l, __uint_as_float(o[j2 + 1]) * inv_l);
            v4.y = pack_bf16x2(__uint_as_float(o[j2 + 2]) * inv_l, __uint_as_float(o[j2 + 3]) * inv_l);
            v4.z = pack_bf16x2(__uint_as_float(o[j2 + 4]) * inv_l, __uint_as_float(o[j2 + 5]) * inv_l);
            v4.w = pack_bf16x2(__uint_as_float(o[j2 + 6]) * inv_l, __uint_as_float(o[j2 + 7]) * inv_l);
            *reinterpret_cast<uint4*>(orow + c + j2) = v4;
          }
        }
      }
      if (valid && a.lse != nullptr)
        a.lse[((int64_t)w.b * a.Hq + h) * a.Sq + qrow] = st.l > 0.f ? (st.m + __log2f(st.l)) * kLn2 : NEG_INF;
    } else {
      // Merge the two halves of the split held by the subtiles, then write
      // the normalised partial O_i and LSE_i for this split.
      if (s == 1) {
        merge_m[row] = st.m;
        merge_l[row] = st.l;
      }
      asm volatile("bar.sync 1, 256;" ::: "memory");
      if (s == 0) {
        const float m1 = merge_m[row], l1v = merge_l[row];
        const float M = fmaxf(st.m, m1);
        const float a0 = (M == NEG_INF || st.m == NEG_INF) ? 0.f : ex2(st.m - M);
        const float a1 = (M == NEG_INF || m1 == NEG_INF) ? 0.f : ex2(m1 - M);
        const float Lsum = st.l * a0 + l1v * a1;
        const float inv = Lsum > 0.f ? 1.0f / Lsum : 0.f;
        const float w0 = a0 * inv, w1 = a1 * inv;
        const int h = w.head[0] + row;
        const bool valid = row < a.g;
        const int64_t prow = ((int64_t)w.b * a.Hq + h) * a.n_splits + w.split;
        const uint32_t tO1 = lane_base + 256 + L::kOCols;
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          uint32_t o0[32], o1[32];
          if (n > 0 && ok) {
            tmem_ld32(tO + c, o0);
            tmem_ld32(tO1 + c, o1);
            tmem_ld_wait();
            reg_fence(o0);
            reg_fence(o1);
          } else {
#pragma unroll
            for (int j2 = 0; j2 < 32; ++j2) o0[j2] = o1[j2] = 0u;
          }
          if (valid) {
            float* dst = a.part_o + prow * D + c;
#pragma unroll
            for (int j2 = 0; j2 < 32; j2 += 4) {
              float4 f;
              f.x = __uint_as_float(o0[j2 + 0]) * w0 + __uint_as_float(o1[j2 + 0]) * w1;
              f.y = __uint_as_float(o0[j2 + 1]) * w0 + __uint_as_float(o1[j2 + 1]) * w1;
              f.z = __uint_as_float(o0[j2 + 2]) * w0 + __uint_as_float(o1[j2 + 2]) * w1;
              f.w = __uint_as_float(o0[j2 + 3]) * w0 + __uint_as_float(o1[j2 + 3]) * w1;
              *reinterpret_cast<float4*>(dst + j2) = f;
            }
          }
        }
        if (valid) a.part_lse[prow] = Lsum > 0.f ? (M + __log2f(Lsum)) * kLn2 : NEG_INF;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) {
    __syncwarp();
    tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0 && bar.abort_flag && a.status) atomicOr(a.status, DEV_TIMEOUT);
}

}  // namespace attn_kernels
