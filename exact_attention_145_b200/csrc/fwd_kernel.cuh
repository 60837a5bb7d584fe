// fwd_kernel.cuh - the attention forward kernel for sm_100a, shared by the
// prefill path (attn_fwd) and the split-KV paged decode path (attn_decode).
//
// One CTA owns two 128-row query sub-tiles ("subtiles" 0 and 1) and streams
// 128-key K/V tiles through shared memory. Warp roles (384 threads):
//   warps 0-3   softmax for subtile 0 (thread t owns query row t = TMEM lane t)
//   warps 4-7   softmax for subtile 1
//   warp  8     tcgen05 MMA issue (one elected lane); owns the TMEM allocation
//   warp  9     TMA producer (one elected lane)
//   warps 10-11 idle (they complete the third warpgroup for the register split)
// The softmax warpgroups raise their register budget to kSoftmaxRegs and the
// third warpgroup lowers its own to kControlRegs: 2*128*224 + 128*56 equals
// the 384*168 registers the block is launched with.
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
constexpr int kThreads = 384;
constexpr int kSoftmaxRegs = 224;
constexpr int kControlRegs = 56;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kControlRegs <= kThreads * 168, "register split exceeds launch budget");
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
  int n_units;     // work units in total; the persistent CTAs walk them
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
  uint64_t q_full, q_empty;
  uint64_t k_full[6];
  uint64_t v_full[6];
  uint64_t kv_empty[6];
  uint64_t s_ready[2];
  uint64_t p_ready[2];
  uint64_t o_done[2];
  uint64_t o_free[2];
  uint64_t merge_full, merge_empty;  // decode: subtile-1 row stats handed to subtile 0
  uint64_t final_mma;
  uint32_t tmem_base;
  int abort_flag;
};

// ---------------------------------------------------------------- work map
struct Work {
  int b, hk;
  int head0, head1;  // query head of each subtile (prefill) / first head of the group (decode)
  int row00, row01;  // first query row of each subtile (prefill)
  int split;    // decode
  int t_begin, t_end;  // decode: key tiles [t_begin, t_end) of this split
  int seqlen;          // decode
};

// Subtile accessors written as selects so the work record stays in registers.
__device__ __forceinline__ int w_head(const Work& w, int s) { return s ? w.head1 : w.head0; }
__device__ __forceinline__ int w_row0(const Work& w, int s) { return s ? w.row01 : w.row00; }

template <bool DECODE>
__device__ __forceinline__ Work map_work(const FwdArgs& a, int u) {
  Work w;
  if constexpr (DECODE) {
    w.split = u % a.n_splits;
    const int bh = u / a.n_splits;
    w.hk = bh % a.Hkv;
    w.b = bh / a.Hkv;
    w.head0 = w.head1 = w.hk * a.g;
    w.row00 = w.row01 = 0;
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
      w.head0 = 2 * hu;
      w.head1 = 2 * hu + 1;
      w.row00 = w.row01 = rt * kRows;
    } else {
      w.head0 = w.head1 = hu;
      w.row00 = 2 * rt * kRows;
      w.row01 = w.row00 + kRows;
    }
    w.hk = w.head0 / a.g;
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
    const int r0 = w_row0(w, s);
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

// The key tiles a work unit visits. Prefill visits every kv tile that is
// non-empty for either subtile, in ascending order: a contiguous range for the
// analytic masks, a scan of the block-mask table otherwise. Decode step i
// gives subtile s the tile t_begin + 2i + s.
struct TileSeq {
  int first;  // first tile (prefill) / t_begin (decode)
  int n;      // number of steps
};

__device__ __forceinline__ bool union_nonempty(const FwdArgs& a, const Work& w, int t) {
  return (tile_class<false>(a, w, 0, t) | tile_class<false>(a, w, 1, t)) != 0;
}

// Tile range [lo, hi] of the window form q_pos - left <= kv <= q_pos + right
// for the valid rows of subtile s; returns false when empty.
__device__ __forceinline__ bool subtile_range(const FwdArgs& a, const Work& w, int s, int& lo, int& hi) {
  const int r0 = w_row0(w, s);
  if (r0 >= a.Sq) return false;
  const long r1 = min(r0 + kRows, a.Sq) - 1;
  long kv_lo = 0, kv_hi = (long)a.Skv - 1;
  if (a.mask != MASK_NONE) {
    if (a.wl >= 0) kv_lo = max(kv_lo, (long)r0 + a.q_offset - a.wl);
    if (a.wr >= 0) kv_hi = min(kv_hi, r1 + a.q_offset + a.wr);
  }
  if (kv_hi < kv_lo) return false;
  lo = (int)(kv_lo / kKeys);
  hi = (int)(kv_hi / kKeys);
  return true;
}

template <bool DECODE>
__device__ __forceinline__ TileSeq tile_seq(const FwdArgs& a, const Work& w) {
  TileSeq ts;
  if constexpr (DECODE) {
    ts.first = w.t_begin;
    ts.n = (w.t_end - w.t_begin + 1) / 2;
  } else if (a.bm_cls == nullptr) {
    int lo0 = 0, hi0 = -1, lo1 = 0, hi1 = -1;
    const bool e0 = subtile_range(a, w, 0, lo0, hi0), e1 = subtile_range(a, w, 1, lo1, hi1);
    if (!e0 && !e1) {
      ts.first = 0;
      ts.n = 0;
    } else {
      // the two subtile ranges overlap or touch (rows differ by at most one tile)
      const int lo = e0 ? (e1 ? min(lo0, lo1) : lo0) : lo1;
      const int hi = e0 ? (e1 ? max(hi0, hi1) : hi0) : hi1;
      ts.first = lo;
      ts.n = hi - lo + 1;
    }
  } else {
    ts.first = a.nK;
    ts.n = 0;
    for (int t = a.nK - 1; t >= 0; --t)
      if (union_nonempty(a, w, t)) {
        ts.first = t;
        ++ts.n;
      }
  }
  return ts;
}

// Next prefill tile after t.
__device__ __forceinline__ int next_tile(const FwdArgs& a, const Work& w, int t) {
  ++t;
  if (a.bm_cls != nullptr)
    while (t < a.nK && !union_nonempty(a, w, t)) ++t;
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

// 2^x on the FMA pipe, to take part of the exponentials off the SFU (which
// would otherwise bound the softmax: 16 results per clock per SM). Cody-Waite
// style range reduction with a round-to-nearest "magic number" add,
// x = n + f with f in [-1/2, 1/2], 2^x = 2^n * q(f), and 2^n applied by
// adding n to the exponent field. q is our own degree-3 fit of 2^f on
// [-1/2, 1/2] with q(0) = 1 (max relative error 1.02e-4, far below the bf16
// rounding P gets anyway). Inputs are clamped at -127, where the result is
// exactly +0, so masked (-inf) entries still contribute exactly nothing.
constexpr float kExp2C1 = 0.693282866192005f;
constexpr float kExp2C2 = 0.24220984271597695f;
constexpr float kExp2C3 = 0.05500836139945104f;
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23

__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  x.x = fmaxf(x.x, -127.0f);
  x.y = fmaxf(x.y, -127.0f);
  const float2 t = add2(x, make_float2(kRoundMagic, kRoundMagic));        // n in the low mantissa bits
  const float2 r = add2(t, make_float2(-kRoundMagic, -kRoundMagic));      // n as a float
  const float2 f = fma2(r, make_float2(-1.f, -1.f), x);                   // x - n
  float2 q = fma2(f, make_float2(kExp2C3, kExp2C3), make_float2(kExp2C2, kExp2C2));
  q = fma2(q, f, make_float2(kExp2C1, kExp2C1));
  q = fma2(q, f, make_float2(1.f, 1.f));
  // n << 23 equals the bits of t shifted left by 23 (the magic's own bits vanish).
  return make_float2(__uint_as_float(__float_as_uint(q.x) + (__float_as_uint(t.x) << 23)),
                     __uint_as_float(__float_as_uint(q.y) + (__float_as_uint(t.y) << 23)));
}
// Which of the 32 column pairs of a half-tile take the FMA-pipe exponential.
__device__ __forceinline__ constexpr bool exp_on_fma(int j) { return (j % 16) >= 9; }

// tanh on the FMA pipe for |y| <= kTanhPolyMax: the Taylor series
// y - y^3/3 + 2y^5/15 - 17y^7/315 + 62y^9/2835 (tail below 1e-7 there).
constexpr float kTanhPolyMax = 0.35f;
constexpr float kTanhA3 = -1.0f / 3.0f;
constexpr float kTanhA5 = 2.0f / 15.0f;
constexpr float kTanhA7 = -17.0f / 315.0f;
constexpr float kTanhA9 = 62.0f / 2835.0f;

// Turns the raw scores of one row into log2-domain scores for the score mods.
// softcap:  x = c*log2(e) * tanh(s*scale/c);  alibi: x = s*scale*log2(e) + slope*log2(e)*(kv - q_pos)
template <bool DECODE, int MOD>
__device__ __forceinline__ void apply_score_mod(const FwdArgs& a, const Work& w, int s, int row, int t, float* x) {
  if constexpr (MOD == MOD_SOFTCAP) {
    const float k1 = a.scale / a.softcap;
    const float cl = a.softcap * kLog2e;
    float smax = 0.f;
#pragma unroll
    for (int c = 0; c < kKeys; c += 2) smax = max3(smax, fabsf(x[c]), fabsf(x[c + 1]));
    if (smax * k1 <= kTanhPolyMax) {
      const float2 K1 = make_float2(k1, k1), CL = make_float2(cl, cl);
      const float2 A3 = make_float2(kTanhA3, kTanhA3), A5 = make_float2(kTanhA5, kTanhA5);
      const float2 A7 = make_float2(kTanhA7, kTanhA7), A9 = make_float2(kTanhA9, kTanhA9);
      const float2 ONE = make_float2(1.f, 1.f);
#pragma unroll
      for (int c = 0; c < kKeys; c += 2) {
        const float2 y = mul2(make_float2(x[c], x[c + 1]), K1);
        const float2 y2 = mul2(y, y);
        float2 q = fma2(y2, A9, A7);
        q = fma2(y2, q, A5);
        q = fma2(y2, q, A3);
        q = fma2(y2, q, ONE);
        const float2 r = mul2(mul2(y, CL), q);
        x[c] = r.x;
        x[c + 1] = r.y;
      }
    } else {
      // Some score of this row is large: tanh(y) = 1 - 2 / (e^{2y} + 1) on the SFU.
      const float k2 = 2.0f * k1 * kLog2e;
#pragma unroll
      for (int c = 0; c < kKeys; ++c) x[c] = cl * (1.0f - 2.0f * rcp(ex2(x[c] * k2) + 1.0f));
    }
  } else if constexpr (MOD == MOD_ALIBI) {
    const long q_pos = DECODE ? (long)w.seqlen - 1 : (long)(w_row0(w, s) + row) + a.q_offset;
    const int head = w_head(w, s) + (DECODE ? row : 0);
    const float slope = a.alibi[(int64_t)w.b * a.alibi_bstride + min(head, a.Hq - 1)] * kLog2e;
    const float base = slope * (float)((long)t * kKeys - q_pos);
    const float2 SC = make_float2(a.scale_log2, a.scale_log2), SL = make_float2(slope, slope);
    const float2 B = make_float2(base, base);
#pragma unroll
    for (int c = 0; c < kKeys; c += 2) {
      const float2 bias = fma2(SL, make_float2((float)c, (float)(c + 1)), B);
      const float2 r = fma2(make_float2(x[c], x[c + 1]), SC, bias);
      x[c] = r.x;
      x[c + 1] = r.y;
    }
  }
}

// Sets disallowed entries of a partial tile to -inf (works on raw or log2-domain scores).
template <bool DECODE>
__device__ __forceinline__ void apply_mask(const FwdArgs& a, const Work& w, int s, int row, int t, float* x) {
  const float NEG_INF = -__int_as_float(0x7f800000);
  const int kv0 = t * kKeys;
  if constexpr (DECODE) {
#pragma unroll
    for (int c = 0; c < kKeys; ++c)
      if (kv0 + c >= w.seqlen) x[c] = NEG_INF;
  } else {
    const int qrow = w_row0(w, s) + row;
    const long q_pos = (long)qrow + a.q_offset;
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
      // allowed iff lo <= kv <= hi, with kv < Skv; as offsets from kv0 in int
      const long lo = a.wl >= 0 ? q_pos - a.wl : -(1l << 40);
      const long hi = min(a.wr >= 0 ? q_pos + a.wr : (1l << 40), (long)Skv - 1);
      const int clo = (int)max(min(lo - kv0, (long)kKeys), -1l);
      const int chi = (int)max(min(hi - kv0, (long)kKeys), -1l);
#pragma unroll
      for (int c = 0; c < kKeys; ++c)
        if (c < clo || c > chi) x[c] = NEG_INF;
    }
  }
}

// Exponentials of one 32-column chunk (16 pairs) against reference max -nmu,
// packed to bf16 pairs; sums and the chunk max are accumulated on the way.
__device__ __forceinline__ void exp_chunk(const float* x, float2 MULT, float2 NMU, uint32_t* pk, float2& acc0,
                                          float2& acc1) {
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const float2 arg = fma2(make_float2(x[2 * j], x[2 * j + 1]), MULT, NMU);
    float2 e;
    if (exp_on_fma(j)) {
      e = exp2_poly2(arg);
    } else {
      e.x = ex2(arg.x);
      e.y = ex2(arg.y);
    }
    if (j & 1)
      acc1 = add2(acc1, e);
    else
      acc0 = add2(acc0, e);
    pk[j] = pack_bf16x2(e.x, e.y);
  }
}

__device__ __forceinline__ float chunk_max(const float* x) {
  float m0 = max3(x[0], x[1], x[2]), m1 = max3(x[3], x[4], x[5]);
#pragma unroll
  for (int c = 6; c < 30; c += 4) {
    m0 = max3(m0, x[c], x[c + 1]);
    m1 = max3(m1, x[c + 2], x[c + 3]);
  }
  return max3(m0, m1, fmaxf(x[30], x[31]));
}

// One key tile of the online softmax for one query row (this thread's TMEM
// lane). The exponentials are taken optimistically against the row's current
// reference max while the scores stream in from TMEM chunk by chunk; only if
// some row of the warp finds a max more than 8 above its reference (always on
// the first tile) is the tile redone against the new max, with O rescaled.
template <int D, bool DECODE, int MOD>
__device__ __forceinline__ void softmax_step(const FwdArgs& a, const Work& w, int s, int row, int t, int cls,
                                             uint32_t tS, uint32_t tO, bool first, RowState& st,
                                             uint64_t* p_ready) {
  float x[kKeys];
  const float NEG_INF = -__int_as_float(0x7f800000);
  const float mult = MOD == MOD_NONE ? a.scale_log2 : 1.0f;  // x * mult is the log2-domain score
  const float2 MULT = make_float2(mult, mult);
  float2 acc0 = make_float2(0.f, 0.f), acc1 = acc0;
  float mt;
  const bool have_ref = !first && __all_sync(0xffffffffu, st.m != NEG_INF);
  const float nmu0 = have_ref ? -st.m : 0.0f;
  if (cls == 0) {
#pragma unroll
    for (int c = 0; c < kKeys; ++c) x[c] = NEG_INF;
    mt = NEG_INF;
    uint32_t pk[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) pk[j] = 0u;
    tmem_st32(tS, pk);
    tmem_st32(tS + 32, pk);
  } else if (MOD == MOD_NONE && cls == 2 && have_ref) {
    // Streamed: chunk c+1 is in flight while chunk c is exponentiated.
    const float2 NMU = make_float2(nmu0, nmu0);
    float mc = NEG_INF;
    tmem_ld32f(tS, x);
    tmem_ld_wait();
    reg_fence_f<32>(x);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      if (c < 3) tmem_ld32f(tS + 32 * (c + 1), x + 32 * (c + 1));
      uint32_t pk[16];
      exp_chunk(x + 32 * c, MULT, NMU, pk, acc0, acc1);
      mc = fmaxf(mc, chunk_max(x + 32 * c));
      tmem_st16(tS + 16 * c, pk);
      if (c < 3) {
        tmem_ld_wait();
        reg_fence_f<32>(x + 32 * (c + 1));
      }
    }
    mt = mc * mult;
  } else {
    tmem_ld128f(tS, x);
    tmem_ld_wait();
    reg_fence_f<kKeys>(x);
    if constexpr (MOD != MOD_NONE) apply_score_mod<DECODE, MOD>(a, w, s, row, t, x);
    if (cls == 1) apply_mask<DECODE>(a, w, s, row, t, x);
    float mc = NEG_INF;
#pragma unroll
    for (int c = 0; c < 4; ++c) mc = fmaxf(mc, chunk_max(x + 32 * c));
    mt = mc * mult;
    if (have_ref) {
      const float2 NMU = make_float2(nmu0, nmu0);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
        exp_chunk(x + 32 * c, MULT, NMU, pk, acc0, acc1);
        tmem_st16(tS + 16 * c, pk);
      }
    }
  }
  // Slow path: first tile of the row, or a max that grew past the threshold.
  const bool grow = !have_ref || mt > st.m + kRescaleThreshold;
  float alpha = 1.0f;
  if (__any_sync(0xffffffffu, grow) && cls != 0) {
    const float m_new = fmaxf(st.m, mt);
    alpha = (m_new == NEG_INF || st.m == NEG_INF) ? (st.m == NEG_INF ? 0.0f : 1.0f) : ex2(st.m - m_new);
    st.m = m_new;
    const float nmu = (m_new == NEG_INF) ? 0.0f : -m_new;
    const float2 NMU = make_float2(nmu, nmu);
    acc0 = acc1 = make_float2(0.f, 0.f);
    tmem_st_wait();  // the optimistic P stores (if any) land before they are overwritten
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t pk[16];
      exp_chunk(x + 32 * c, MULT, NMU, pk, acc0, acc1);
      tmem_st16(tS + 16 * c, pk);
    }
    if (!first) {
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
        for (int j = 0; j < 32; j += 2) {
          const float2 r = mul2(make_float2(o[j], o[j + 1]), make_float2(alpha, alpha));
          ob[j] = __float_as_uint(r.x);
          ob[j + 1] = __float_as_uint(r.y);
        }
        tmem_st32(tO + c, ob);
      }
    }
  }
  tmem_st_wait();
  tc_fence_before();
  mbar_arrive(p_ready);
  acc0 = add2(acc0, acc1);
  st.l = st.l * alpha + (acc0.x + acc0.y);
}

// ---------------------------------------------------------------- kernel
// Epilogue of one unit for softmax subtile s: O / l to bf16 (prefill) or the
// merged, normalised split partial (decode), and the LSE.
template <int D, bool DECODE>
__device__ __forceinline__ bool epilogue(const FwdArgs& a, const Work& w, int s, int row, uint32_t lane_base,
                                         bool have_o, const RowState& st, float* merge_m, float* merge_l,
                                         Barriers& bar, int mcnt, volatile int* abort_flag) {
  using L = Layout<D, DECODE>;
  const float NEG_INF = -__int_as_float(0x7f800000);
  const uint32_t tO = lane_base + 256 + s * L::kOCols;
  if constexpr (!DECODE) {
    const int qrow = w_row0(w, s) + row;
    const int h = w_head(w, s);
    const bool valid = qrow < a.Sq && w_row0(w, s) < a.Sq;
    const float inv_l = st.l > 0.f ? 1.0f / st.l : 0.f;
    __nv_bfloat16* orow = a.o + (int64_t)w.b * a.o_sb + (int64_t)qrow * a.o_ss + (int64_t)h * a.o_sh;
#pragma unroll
    for (int c = 0; c < D; c += 32) {
      float o[32];
      if (have_o) {
        tmem_ld32f(tO + c, o);
        tmem_ld_wait();
        reg_fence_f<32>(o);
      } else {
#pragma unroll
        for (int j2 = 0; j2 < 32; ++j2) o[j2] = 0.f;
      }
      if (valid) {
#pragma unroll
        for (int j2 = 0; j2 < 32; j2 += 8) {
          uint4 v4;
          v4.x = pack_bf16x2(o[j2 + 0] * inv_l, o[j2 + 1] * inv_l);
          v4.y = pack_bf16x2(o[j2 + 2] * inv_l, o[j2 + 3] * inv_l);
          v4.z = pack_bf16x2(o[j2 + 4] * inv_l, o[j2 + 5] * inv_l);
          v4.w = pack_bf16x2(o[j2 + 6] * inv_l, o[j2 + 7] * inv_l);
          *reinterpret_cast<uint4*>(orow + c + j2) = v4;
        }
      }
    }
    if (valid && a.lse != nullptr)
      a.lse[((int64_t)w.b * a.Hq + h) * a.Sq + qrow] = st.l > 0.f ? (st.m + __log2f(st.l)) * kLn2 : NEG_INF;
    (void)bar;
    (void)mcnt;
    (void)abort_flag;
  } else {
    // Merge the two halves of the split held by the subtiles, then write the
    // normalised partial O_i and LSE_i of this split. The row stats of
    // subtile 1 are handed over through shared memory with two bounded
    // mbarrier handshakes (no named barrier, so an abort cannot hang here).
    float m1 = NEG_INF, l1v = 0.f;
    if (have_o) {
      if (s == 1) {
        if (mcnt > 0 && !__all_sync(0xffffffffu, mbar_wait(&bar.merge_empty, (mcnt - 1) & 1, abort_flag)))
          return false;
        merge_m[row] = st.m;
        merge_l[row] = st.l;
        mbar_arrive(&bar.merge_full);
        return true;
      }
      if (!__all_sync(0xffffffffu, mbar_wait(&bar.merge_full, mcnt & 1, abort_flag))) return false;
      m1 = merge_m[row];
      l1v = merge_l[row];
      mbar_arrive(&bar.merge_empty);
    }
    if (s == 0) {
      const float M = fmaxf(st.m, m1);
      const float a0 = (M == NEG_INF || st.m == NEG_INF) ? 0.f : ex2(st.m - M);
      const float a1 = (M == NEG_INF || m1 == NEG_INF) ? 0.f : ex2(m1 - M);
      const float Lsum = st.l * a0 + l1v * a1;
      const float inv = Lsum > 0.f ? 1.0f / Lsum : 0.f;
      const float w0 = a0 * inv, w1 = a1 * inv;
      const int h = w.head0 + row;
      const bool valid = row < a.g;
      const int64_t prow = ((int64_t)w.b * a.Hq + h) * a.n_splits + w.split;
      const uint32_t tO1 = lane_base + 256 + L::kOCols;
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        float o0[32], o1[32];
        if (have_o) {
          tmem_ld32f(tO + c, o0);
          tmem_ld32f(tO1 + c, o1);
          tmem_ld_wait();
          reg_fence_f<32>(o0);
          reg_fence_f<32>(o1);
        } else {
#pragma unroll
          for (int j2 = 0; j2 < 32; ++j2) o0[j2] = o1[j2] = 0.f;
        }
        if (valid) {
          float* dst = a.part_o + prow * D + c;
#pragma unroll
          for (int j2 = 0; j2 < 32; j2 += 4) {
            float4 f;
            f.x = o0[j2 + 0] * w0 + o1[j2 + 0] * w1;
            f.y = o0[j2 + 1] * w0 + o1[j2 + 1] * w1;
            f.z = o0[j2 + 2] * w0 + o1[j2 + 2] * w1;
            f.w = o0[j2 + 3] * w0 + o1[j2 + 3] * w1;
            *reinterpret_cast<float4*>(dst + j2) = f;
          }
        }
      }
      if (valid) a.part_lse[prow] = Lsum > 0.f ? (M + __log2f(Lsum)) * kLn2 : NEG_INF;
    }
  }
  return true;
}

// Persistent kernel: CTA c walks the work units c, 2G-1-c, 2G+c, ... (G CTAs,
// units ordered heaviest first), keeping its TMEM allocation, barriers and
// K/V ring across units. Barrier phases count events across units:
//   q_full / q_empty / o_done / o_free   once per unit that has key tiles,
//   s_ready / p_ready                     once per step,
//   k_full / v_full / kv_empty            once per K/V load.
// While the softmax warps write a unit's outputs, the producer already loads
// the next unit's Q and K/V and the MMA warp runs its first QK^T products.
template <int D, bool DECODE, int MOD>
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

  if (threadIdx.x == 0) {
    bar.abort_flag = 0;
    mbar_init(&bar.q_full, 1);
    mbar_init(&bar.q_empty, 1);
    for (int i = 0; i < L::kNSlot; ++i) {
      mbar_init(&bar.k_full[i], 1);
      mbar_init(&bar.v_full[i], 1);
      mbar_init(&bar.kv_empty[i], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar.s_ready[s], 1);
      mbar_init(&bar.p_ready[s], 128);
      mbar_init(&bar.o_done[s], 1);
      mbar_init(&bar.o_free[s], 128);
    }
    mbar_init(&bar.merge_full, 128);
    mbar_init(&bar.merge_empty, 128);
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

  const int G = gridDim.x;
  const int rounds = (a.n_units + G - 1) / G;
  auto unit_of = [&](int r) -> int {
    const int c = (r & 1) ? G - 1 - (int)blockIdx.x : (int)blockIdx.x;
    const int u = r * G + c;
    return u < a.n_units ? u : -1;
  };
  auto wait_all = [&](uint64_t* b, uint32_t par) {
    const bool got = mbar_wait(b, par, abort_flag);
    return __all_sync(0xffffffffu, got);
  };

  if (warp == kTmaWarp) {
    regs_decrease<kControlRegs>();
    // ------------------------------------------------------------ producer
    if (elect_one_sync()) {
      tma_prefetch_desc(&map_q);
      tma_prefetch_desc(&map_k);
      tma_prefetch_desc(&map_v);
    }
    __syncwarp();
    int kload = 0;  // K/V loads issued so far: ring position and phase
    int qcnt = 0;   // units with key tiles so far
    bool ok = true;
    for (int r = 0; ok && r < rounds; ++r) {
      const int u = unit_of(r);
      if (u < 0) continue;
      const Work w = map_work<DECODE>(a, u);
      const TileSeq ts = tile_seq<DECODE>(a, w);
      if (ts.n == 0) continue;
      if (qcnt > 0 && !wait_all(&bar.q_empty, (qcnt - 1) & 1)) {
        ok = false;
        break;
      }
      if (elect_one_sync()) {
        mbar_arrive_expect_tx(&bar.q_full, L::kNQ * L::kTileBytes);
        for (int s = 0; s < L::kNQ; ++s)
          for (int c = 0; c < D / 64; ++c) {
            uint8_t* dst = smem + L::kQOff + s * L::kTileBytes + c * L::kChunk;
            if constexpr (DECODE)
              tma_load_3d(dst, &map_q, &bar.q_full, c * 64, w.head0, w.b);
            else
              tma_load_4d(dst, &map_q, &bar.q_full, c * 64, w_row0(w, s), w_head(w, s), w.b);
          }
      }
      __syncwarp();
      ++qcnt;
      const int n_loads = DECODE ? 2 * ts.n : ts.n;
      int t = ts.first;
      for (int k = 0; k < n_loads; ++k) {
        const int slot = kload % L::kNSlot;
        const int use = kload / L::kNSlot;
        if (use > 0 && !wait_all(&bar.kv_empty[slot], (use - 1) & 1)) {
          ok = false;
          break;
        }
        const bool absent = DECODE && t >= w.t_end;
        if (elect_one_sync())
          load_kv_tile<D, DECODE>(a, w, &map_k, &map_v, smem + L::kKOff + slot * L::kTileBytes,
                                  smem + L::kVOff + slot * L::kTileBytes, &bar.k_full[slot], &bar.v_full[slot], t,
                                  absent);
        __syncwarp();
        ++kload;
        t = DECODE ? t + 1 : next_tile(a, w, t);
      }
    }
    // Drain: on an abort, wait (bounded) for every copy still in flight so
    // none lands in shared memory after the CTA has exited.
    if (*abort_flag) {
      for (int k = max(0, kload - L::kNSlot); k < kload; ++k) {
        const int slot = k % L::kNSlot;
        const uint32_t par = (k / L::kNSlot) & 1;
        mbar_wait_timeout(&bar.k_full[slot], par);
        mbar_wait_timeout(&bar.v_full[slot], par);
      }
      if (qcnt > 0) mbar_wait_timeout(&bar.q_full, (qcnt - 1) & 1);
    }
  } else if (warp == kMmaWarp) {
    regs_decrease<kControlRegs>();
    // ------------------------------------------------------------ MMA issue
    constexpr uint32_t idesc_qk = idesc_bf16_f32(128, kKeys, 0, 0);
    constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
    // Descriptor low words (start address in 16-byte units + LBO); every
    // per-MMA offset below is a compile-time constant added to them.
    constexpr uint32_t kHi = sdesc_sw128_hi(1024);
    const uint32_t q_lo = sdesc_sw128_lo(smem_u32(smem + L::kQOff), 16);
    const uint32_t k_lo = sdesc_sw128_lo(smem_u32(smem + L::kKOff), 16);
    const uint32_t v_lo = sdesc_sw128_lo(smem_u32(smem + L::kVOff), L::kChunk);
    constexpr uint32_t kTileUnits = L::kTileBytes >> 4;
    auto issue_qk = [&](int s, int slot) {
      const uint32_t qa = q_lo + (DECODE ? 0u : (uint32_t)s * kTileUnits);
      const uint32_t ka = k_lo + (uint32_t)slot * kTileUnits;
      if (elect_one_sync()) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk / 4) * L::kChunk + (kk % 4) * 32) >> 4;
          mma_ss(tmem + s * 128, sdesc_join(qa + off, kHi), sdesc_join(ka + off, kHi), idesc_qk, kk > 0);
        }
        mma_commit(&bar.s_ready[s]);
      }
      __syncwarp();
    };
    auto slot_of = [&](int g, int s) { return DECODE ? (2 * g + s) % L::kNSlot : g % L::kNSlot; };
    auto phase_of = [&](int g, int s) { return (uint32_t)(((DECODE ? 2 * g + s : g) / L::kNSlot) & 1); };
    int gstep = 0;  // steps issued so far across units
    int qcnt = 0;   // units with key tiles so far
    bool ok = true;
    for (int r = 0; ok && r < rounds; ++r) {
      const int u = unit_of(r);
      if (u < 0) continue;
      const Work w = map_work<DECODE>(a, u);
      const TileSeq ts = tile_seq<DECODE>(a, w);
      const int n = ts.n;
      if (n == 0) continue;
      ok = wait_all(&bar.q_full, qcnt & 1);
      if (ok) ok = wait_all(&bar.k_full[slot_of(gstep, 0)], phase_of(gstep, 0));
      if (ok) {
        tc_fence_after();
        issue_qk(0, slot_of(gstep, 0));
        if (DECODE) ok = wait_all(&bar.k_full[slot_of(gstep, 1)], phase_of(gstep, 1));
        tc_fence_after();
        if (ok) issue_qk(1, slot_of(gstep, 1));
      }
      for (int j = 0; ok && j < n; ++j) {
        const int g = gstep + j;
        const bool more = j + 1 < n;
#pragma unroll
        for (int s = 0; s < 2; ++s) {
          const int slot = slot_of(g, s);
          if (!wait_all(&bar.v_full[slot], phase_of(g, s))) { ok = false; break; }
          if (!wait_all(&bar.p_ready[s], g & 1)) { ok = false; break; }
          // The first PV of a unit overwrites O(s): the previous unit's epilogue must have read it.
          if (j == 0 && qcnt > 0 && !wait_all(&bar.o_free[s], (qcnt - 1) & 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t va = v_lo + (uint32_t)slot * kTileUnits;
          if (elect_one_sync()) {
#pragma unroll
            for (int kk = 0; kk < kKeys / 16; ++kk)
              mma_ts(tmem + 256 + s * L::kOCols, tmem + s * 128 + kk * 8,
                     sdesc_join(va + ((kk * 16 * 128) >> 4), kHi), idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
            if (!more) mma_commit(&bar.o_done[s]);
            if (DECODE || s == 1) mma_commit(&bar.kv_empty[slot]);
            if (!more && s == 1) mma_commit(&bar.q_empty);  // every QK^T of the unit precedes
          }
          __syncwarp();
          if (more) {
            const int nslot = slot_of(g + 1, s);
            if (!wait_all(&bar.k_full[nslot], phase_of(g + 1, s))) { ok = false; break; }
            tc_fence_after();
            issue_qk(s, nslot);
          }
        }
      }
      gstep += n;
      ++qcnt;
    }
    // Every MMA must be complete before TMEM is released.
    if (elect_one_sync()) mma_commit(&bar.final_mma);
    __syncwarp();
    mbar_wait_timeout(&bar.final_mma, 0);
  } else if (warp >= 10) {
    regs_decrease<kControlRegs>();
  } else {
    regs_increase<kSoftmaxRegs>();
    // ------------------------------------------------------------ softmax
    const int s = warp / 4;
    const int row = threadIdx.x % 128;  // TMEM lane
    const uint32_t lane_base = tmem + ((uint32_t)((warp % 4) * 32) << 16);
    const uint32_t tS = lane_base + s * 128;
    const uint32_t tO = lane_base + 256 + s * L::kOCols;
    int gstep = 0, qcnt = 0;
    bool ok = true;
    for (int r = 0; ok && r < rounds; ++r) {
      const int u = unit_of(r);
      if (u < 0) continue;
      const Work w = map_work<DECODE>(a, u);
      const TileSeq ts = tile_seq<DECODE>(a, w);
      const int n = ts.n;
      RowState st;
      st.m = -__int_as_float(0x7f800000);
      st.l = 0.f;
      if (n == 0) {
        epilogue<D, DECODE>(a, w, s, row, lane_base, false, st, merge_m, merge_l, bar, qcnt, abort_flag);
        continue;
      }
      int t = DECODE ? ts.first + s : ts.first;
      for (int j = 0; j < n; ++j) {
        const int cls = tile_class<DECODE>(a, w, s, t);
        if (!wait_all(&bar.s_ready[s], (gstep + j) & 1)) { ok = false; break; }
        tc_fence_after();
        softmax_step<D, DECODE, MOD>(a, w, s, row, t, cls, tS, tO, j == 0, st, &bar.p_ready[s]);
        t = DECODE ? t + 2 : next_tile(a, w, t);
      }
      if (!ok) break;
      bool got = wait_all(&bar.o_done[s], qcnt & 1);
      if (DECODE && s == 0) got = got && wait_all(&bar.o_done[1], qcnt & 1);
      if (!got) break;
      tc_fence_after();
      if (!epilogue<D, DECODE>(a, w, s, row, lane_base, true, st, merge_m, merge_l, bar, qcnt, abort_flag)) break;
      // O is read: the next unit's first PV may overwrite it. In decode the
      // subtile-0 threads read both accumulators and release both.
      tc_fence_before();
      if (!DECODE) {
        mbar_arrive(&bar.o_free[s]);
      } else if (s == 0) {
        mbar_arrive(&bar.o_free[0]);
        mbar_arrive(&bar.o_free[1]);
      }
      gstep += n;
      ++qcnt;
    }
    (void)tO;
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
