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
// the 384*168 registers the block is launched with. setmaxnreg acts on a whole
// warpgroup: its four warps must all request the same count, so the idle
// warps cannot give their share to the MMA and TMA warps.
// The tensor pipe alternates between the subtiles so that one subtile's
// softmax overlaps the other's MMAs: on B200 the exponentials take about
// twice as long as the two GEMMs of a tile, so a single query tile per CTA
// would leave the tensor cores idle ("FlexAttention + FlashAttention-4" talk,
// the two-Q-tile ping-pong pipeline). MMA order per step, whole tiles
// (decode, and prefill without the softcap):
//   PV(0, j) QK(0, j+1) PV(1, j) QK(1, j+1)
// Prefill with the softcap hands tiles over in key halves a (keys 0-63) and
// b (keys 64-127), see "prefill, half tiles" below:
//   PVa(0) QKa(0) PVa(1) QKa(1) PVb(0) QKb(0) PVb(1) QKb(1)
// TMEM (512 columns): S0 | S1 | O0 | O1. P (bf16) overwrites part of its S
// region once the softmax has read those scores into registers (columns
// [0, 64) for whole tiles; [0, 32) and [64, 96) for half tiles) and feeds the
// PV MMA straight from TMEM. tcgen05.mma ops of one thread execute in issue
// order, so a QK^T overwrites S(s) only after the PV that reads P from it.
//
// Online softmax ("A Deep Dive into Flash Attention", section "2. Online
// Softmax"), in base 2: x = log2(e) * score; each row keeps a reference max
// m and a running sum l; O is rescaled by 2^(m_old - m_new) only when some
// row of the warp sees its max grow by more than 8 (probabilities stay below
// 2^8, which bf16 P and the fp32 accumulators absorb exactly as well).
// With whole tiles QK(s, j+1) is committed after PV(s, j), so seeing
// S(s, j+1) ready implies O(s) is settled and the rescale needs no extra
// wait; half tiles wait for the one PV that may still be in flight.
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
constexpr int kControlRegs = 56;  // warps 8-11, one warpgroup, one count
static_assert(2 * 128 * kSoftmaxRegs + 128 * kControlRegs <= kThreads * 168, "register split exceeds launch budget");
constexpr int kMmaWarp = 8;    // MMA issue for subtile 0; owns the TMEM allocation
constexpr int kTmaWarp = 9;
constexpr int kMmaWarp1 = 10;  // MMA issue for subtile 1 when kMmaWarps == 2
constexpr int kMmaWarps = 1;   // warps issuing MMAs: 1 (both subtiles) or 2 (one each)
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

enum : int { MASK_NONE = 0, MASK_CAUSAL = 1, MASK_WINDOW = 2, MASK_DOCUMENT = 3 };
enum : int { MOD_NONE = 0, MOD_SOFTCAP = 1, MOD_ALIBI = 2, MOD_RELU = 3 };
enum : int { DEV_TIMEOUT = 1, DEV_BAD_PAGE = 2, DEV_BAD_LEN = 4, DEV_BAD_MASK = 8 };

struct FwdArgs {
  int B, Hq, Hkv, Sq, Skv, g;
  float scale_log2;     // softmax scale * log2(e)
  float scale;          // softmax scale
  int mask, wl, wr, q_offset;
  const int32_t* doc_id;
  int64_t doc_bstride;    // elements between the document rows of batches (0: one shared row)
  const uint8_t* bm_cls;  // [Bm][Hm][nQ][nK] class tables or nullptr
  const int32_t *bm_part_cnt, *bm_part_idx, *bm_full_cnt, *bm_full_idx;  // ascending kv-tile lists
  int bm_Bm, bm_Hm;       // slices of the block mask (1 = shared by every batch / head)
  int bm_rows, bm_nQ;     // query rows per table row (128 or 256) and table rows
  const int32_t* bm_row_order;   // [Bm][nQ] q-tiles heaviest first, or nullptr
  const int32_t* bm_doc_start;   // [Bm][Sq] document run starts (document masks)
  const int32_t* bm_doc_sorted;  // [Bm] 1: every document is one run of ids
  int nQ, nK;
  int mod;
  float softcap;
  float softcap_k1;  // scale / softcap (the tanh argument per raw score)
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
  const int32_t* block_table;  // null: contiguous cache, rows cache_batch_idx[b] (or b)
  const int32_t* cache_batch_idx;
  int bt_stride;
  const int32_t* seqlens;
  int page_size, num_pages, box_rows, n_splits, tiles_per_split;
  int max_seqlen;   // upper bound on cache_seqlens[b]; larger lengths are clamped and reported
  // Decode rows: q_len new tokens per sequence x g heads (row r: token r / g,
  // head r % g of the group); with q_causal token i sees the keys below
  // seqlen - (q_len - 1 - i). q_bytes: bytes one Q load brings.
  int q_len, q_causal, q_bytes;
  float* part_o;    // [B][Hq][n_splits][D]
  float* part_lse;  // [B][Hq][n_splits]
  int* status;
  // cycle trace (ATTN_TRACE builds only; null otherwise): per CTA and role,
  // trace_per_role records of {cycles since kernel start, event << 24 | aux}
  uint2* trace;
  int trace_per_role;
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
  // After the barriers: decode's merge scratch (two 128-float rows), or
  // prefill's output staging, one 32-row x 64-column bf16 SW128 box per
  // softmax warp (the source of that warp's TMA stores).
  static constexpr int kExtraOff = kBarOff + 1024;
  static constexpr int kStageWarpBytes = 32 * 128;
  static constexpr int kExtraBytes = DECODE ? 2 * 128 * 4 : 8 * kStageWarpBytes;
  static constexpr int kSmemBytes = kExtraOff + kExtraBytes + 1024;  // + alignment slack
  static constexpr int kOCols = D;  // TMEM columns of one O accumulator
  static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
  static_assert(kExtraOff % 1024 == 0, "SW128 staging needs 1024-byte alignment");
};

struct Barriers {
  uint64_t q_full, q_empty;
  uint64_t k_full[6];
  uint64_t v_full[6];
  uint64_t k_empty[6];    // the K tile of the slot has been read by every QK^T that uses it
  uint64_t v_empty[6];    // the V tile of the slot has been read by every PV that uses it
  uint64_t s_ready[2];    // prefill: keys 0-63 of S ready (decode: the whole S)
  uint64_t p_ready[2];    // prefill: P for keys 0-63 written (decode: the whole P)
  uint64_t s_b_ready[2];  // prefill: keys 64-127 of S ready
  uint64_t p_b_ready[2];  // prefill: P for keys 64-127 written
  uint64_t pv_a_done[2];  // prefill: the PV of keys 0-63 has completed
  uint64_t o_done[2];
  uint64_t o_free[2];
  uint64_t merge_full, merge_empty;  // decode: subtile-1 row stats handed to subtile 0
  uint64_t final_mma[2];
  uint64_t mma_turn[2];   // turn token between the two MMA warps (kMmaWarps == 2)
  uint32_t tmem_base;
  int abort_flag;
  uint32_t trace_cnt[11]; // ATTN_TRACE: records written per role
  long long trace_t0;     // ATTN_TRACE: clock64 at kernel start
};

// ---------------------------------------------------------------- cycle trace
// Compiled in only with -DATTN_TRACE (a separate build of the library): lane
// 0 of each role's warp (role = warp index: softmax warps 0-7, MMA warps 8 and
// 10, TMA warp 9) appends {SM cycles since kernel start, event id << 24 | aux}
// records to the caller's buffer. Normal builds contain none of this.
enum : int {
  kTraceRoles = 11, TR_TMA = 9,
  EV_S_WAIT = 1, EV_S_READY = 2, EV_P_DONE = 3, EV_O_WAIT = 4, EV_EPI_BEGIN = 5, EV_EPI_END = 6,
  EV_HALF_A_DONE = 7, EV_SB_WAIT = 8, EV_SB_READY = 9,
  EV_Q_FULL = 10, EV_PV = 11, EV_QK = 12, EV_P_WAIT = 13, EV_MMA_END = 14, EV_PV_ISSUED = 15,
  EV_Q_LOAD = 20, EV_KV_LOAD = 21, EV_KERNEL_END = 30
};
#ifdef ATTN_TRACE
__device__ __forceinline__ void trace_rec(const FwdArgs& a, Barriers& bar, int role, int ev, int aux) {
  if ((threadIdx.x & 31) == 0 && a.trace != nullptr) {
    const uint32_t n = bar.trace_cnt[role];
    if (n < (uint32_t)a.trace_per_role) {
      a.trace[((size_t)blockIdx.x * kTraceRoles + role) * a.trace_per_role + n] =
          make_uint2((uint32_t)(clock64() - bar.trace_t0), ((uint32_t)ev << 24) | ((uint32_t)aux & 0xffffffu));
      bar.trace_cnt[role] = n + 1;
    }
  }
}
#define ATTN_TRACE_REC(role, ev, aux) trace_rec(a, bar, (role), (ev), (aux))
#else
#define ATTN_TRACE_REC(role, ev, aux) ((void)0)
#endif

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
    // Keys past max_seqlen would fall outside the splits (and possibly the
    // block table); such lengths are clamped here and reported by the producer.
    w.seqlen = min(max(a.seqlens[w.b], 0), a.max_seqlen);
    const int nt = (w.seqlen + kKeys - 1) / kKeys;
    w.t_begin = min(nt, w.split * a.tiles_per_split);
    w.t_end = min(nt, w.t_begin + a.tiles_per_split);
  } else {
    // Heaviest row tiles first: unit index u walks row tiles from the end
    // (the causal and window forms), or in the block mask's work order.
    const int HU = a.pair_heads ? a.Hq / 2 : a.Hq;
    const int per = a.B * HU;
    const int qi = u / per, rem = u % per;
    w.b = rem / HU;
    const int hu = rem % HU;
    int rt = a.n_row_units - 1 - qi;
    if (a.bm_row_order != nullptr && a.pair_heads) {
      // Table rows in the table's order; a 256-row table row expands into
      // its two 128-row tiles (units past the last tile are empty). A
      // caller-written order entry outside the table falls back to the
      // default order (the producer reports it as a bad mask).
      const int sub = a.bm_rows / kRows;
      const int o = __ldg(a.bm_row_order + (int64_t)(a.bm_Bm == 1 ? 0 : w.b) * a.bm_nQ + qi / sub);
      if (o >= 0 && o < a.bm_nQ) rt = o * sub + qi % sub;
    }
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

// Block-mask slice (batch, head) that serves query head h of batch b.
__device__ __forceinline__ int64_t bm_slice(const FwdArgs& a, int b, int h) {
  return (int64_t)(a.bm_Bm == 1 ? 0 : b) * a.bm_Hm + (a.bm_Hm == 1 ? 0 : h);
}

// Tile class of kv tile t for subtile s: 0 empty, 1 partial, 2 full. BM:
// the classes come from a block mask's table instead of the window bounds.
template <bool DECODE, bool BM>
__device__ __forceinline__ int tile_class(const FwdArgs& a, const Work& w, int s, int t) {
  if constexpr (DECODE) {
    (void)s;
    if (t < w.t_begin || t >= w.t_end) return 0;
    return (t + 1) * kKeys <= w.seqlen - (a.q_causal ? a.q_len - 1 : 0) ? 2 : 1;
  } else {
    const int r0 = w_row0(w, s);
    if (r0 >= a.Sq || t < 0 || t >= a.nK) return 0;
    const int r1 = min(r0 + kRows, a.Sq) - 1;
    const int c0 = t * kKeys;
    const int c1 = min(c0 + kKeys, a.Skv) - 1;
    const bool ragged = c0 + kKeys > a.Skv;
    int cls;
    if constexpr (BM) {
      cls = a.bm_cls[(bm_slice(a, w.b, w_head(w, s)) * a.bm_nQ + r0 / a.bm_rows) * a.nK + t];
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

// The key tiles a work unit visits, in ascending order. Prefill visits every
// kv tile that is non-empty for either subtile: a contiguous range for the
// analytic masks, the merge of the two subtiles' partial and full lists when
// a block mask is given. Decode step i gives subtile s the tile t_begin+2i+s.
struct TileWalker {
  int t;  // current tile
  // block-mask lists of the two subtiles' q-tiles (empty for an absent subtile)
  const int32_t *p0, *f0, *p1, *f1;
  int np0, nf0, np1, nf1, ip0, if0, ip1, if1;
};

// Walk order over the key tiles of a unit. Ascending by default; descending
// (from the diagonal back) for prefill with ALiBi, whose bias grows towards
// the query: walked upwards, a row's max would rise by up to slope x 128 per
// tile (log2 units), far past the rescale threshold, and every tile would
// redo its exponentials and rescale O. Walked downwards, the first tiles
// hold the largest biases and later ones rarely exceed them.
template <bool DECODE, int MOD>
constexpr bool kDescWalk = !DECODE && MOD == MOD_ALIBI;
// Prefill softmax with ALiBi: minus the row's reference max joins the bias,
// so the biased scores come out as exponents (one packed op per pair fewer).
template <int MOD>
constexpr bool kFoldRef = MOD == MOD_ALIBI;
constexpr int kWalkEnd = 0x7fffffff;  // walker_peek past the last tile

// Head i of an ascending list of n entries, taken from the front or the back.
template <bool DESC>
__device__ __forceinline__ int list_head(const int32_t* l, int n, int i) {
  if (i >= n) return DESC ? -1 : kWalkEnd;
  return __ldg(l + (DESC ? n - 1 - i : i));
}

template <bool DESC>
__device__ __forceinline__ int walker_peek(const TileWalker& tw) {
  const int a0 = list_head<DESC>(tw.p0, tw.np0, tw.ip0), b0 = list_head<DESC>(tw.f0, tw.nf0, tw.if0);
  const int a1 = list_head<DESC>(tw.p1, tw.np1, tw.ip1), b1 = list_head<DESC>(tw.f1, tw.nf1, tw.if1);
  if constexpr (DESC) {
    const int m = max(max(a0, b0), max(a1, b1));
    return m < 0 ? kWalkEnd : m;
  } else {
    return min(min(a0, b0), min(a1, b1));
  }
}

// Consumes tile t from every list whose head it is.
template <bool DESC>
__device__ __forceinline__ void walker_pop(TileWalker& tw, int t) {
  if (list_head<DESC>(tw.p0, tw.np0, tw.ip0) == t) ++tw.ip0;
  if (list_head<DESC>(tw.f0, tw.nf0, tw.if0) == t) ++tw.if0;
  if (list_head<DESC>(tw.p1, tw.np1, tw.ip1) == t) ++tw.ip1;
  if (list_head<DESC>(tw.f1, tw.nf1, tw.if1) == t) ++tw.if1;
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

// Sets up the walk of one unit; returns the number of steps and leaves
// tw.t on the first tile (the lowest, or the highest with DESC).
template <bool DECODE, bool BM, bool DESC = false>
__device__ __forceinline__ int walker_init(const FwdArgs& a, const Work& w, TileWalker& tw) {
  tw.np0 = tw.nf0 = tw.np1 = tw.nf1 = tw.ip0 = tw.if0 = tw.ip1 = tw.if1 = 0;
  tw.p0 = tw.f0 = tw.p1 = tw.f1 = nullptr;
  if constexpr (DECODE) {
    tw.t = w.t_begin;
    return (w.t_end - w.t_begin + 1) / 2;
  } else if constexpr (!BM) {
    int lo0 = 0, hi0 = -1, lo1 = 0, hi1 = -1;
    const bool e0 = subtile_range(a, w, 0, lo0, hi0), e1 = subtile_range(a, w, 1, lo1, hi1);
    if (!e0 && !e1) {
      tw.t = 0;
      return 0;
    }
    // the two subtile ranges overlap or touch (rows differ by at most one tile)
    const int lo = e0 ? (e1 ? min(lo0, lo1) : lo0) : lo1;
    const int hi = e0 ? (e1 ? max(hi0, hi1) : hi0) : hi1;
    tw.t = DESC ? hi : lo;
    return hi - lo + 1;
  } else {
    // row q-tile of each subtile within its (batch, head) slice; the second
    // list is needed only when the subtiles differ in rows or in slice
    const int64_t q0 = bm_slice(a, w.b, w.head0) * a.bm_nQ + w.row00 / a.bm_rows;
    const int64_t q1 = bm_slice(a, w.b, w.head1) * a.bm_nQ + w.row01 / a.bm_rows;
    // counts are clamped to a row's length, so lists are never read past it
    if (w.row00 < a.Sq) {
      tw.np0 = min(max(__ldg(a.bm_part_cnt + q0), 0), a.nK);
      tw.nf0 = min(max(__ldg(a.bm_full_cnt + q0), 0), a.nK);
      tw.p0 = a.bm_part_idx + q0 * a.nK;
      tw.f0 = a.bm_full_idx + q0 * a.nK;
    }
    if (w.row01 < a.Sq && q1 != q0) {
      tw.np1 = min(max(__ldg(a.bm_part_cnt + q1), 0), a.nK);
      tw.nf1 = min(max(__ldg(a.bm_full_cnt + q1), 0), a.nK);
      tw.p1 = a.bm_part_idx + q1 * a.nK;
      tw.f1 = a.bm_full_idx + q1 * a.nK;
    }
    // count the union, then rewind
    int n = 0;
    TileWalker c = tw;
    for (int t = walker_peek<DESC>(c); t != kWalkEnd; t = walker_peek<DESC>(c)) {
      walker_pop<DESC>(c, t);
      ++n;
    }
    tw.t = walker_peek<DESC>(tw);
    return n;
  }
}

// Advances a prefill walk to the next tile.
template <bool BM, bool DESC = false>
__device__ __forceinline__ void walker_next(TileWalker& tw) {
  if constexpr (!BM) {
    tw.t += DESC ? -1 : 1;
  } else {
    walker_pop<DESC>(tw, tw.t);
    tw.t = walker_peek<DESC>(tw);
  }
}

// ---------------------------------------------------------------- producer
// Loads key tile t of K or of V (map m) into dst, completing on bar.
template <int D, bool DECODE>
__device__ __forceinline__ void load_kv_tile(const FwdArgs& a, const Work& w, const CUtensorMap* m, uint8_t* dst,
                                             uint64_t* bar, int t, bool absent, bool report) {
  using L = Layout<D, DECODE>;
  mbar_arrive_expect_tx(bar, L::kTileBytes);
  if constexpr (DECODE) {
    const int rows = a.box_rows;
    for (int u = 0; u < kKeys / rows; ++u) {
      const int tok = t * kKeys + u * rows;
      const int lp = tok / a.page_size;
      const int slot = tok % a.page_size;
      int phys = a.num_pages;  // out of range -> TMA fills zeros, no memory read
      if (!absent && tok < w.seqlen && lp < a.bt_stride) {
        // contiguous cache (no block table): one "page" per cache row
        const int pg = a.block_table ? a.block_table[(int64_t)w.b * a.bt_stride + lp]
                                     : (a.cache_batch_idx ? a.cache_batch_idx[w.b] : w.b);
        if (pg >= 0 && pg < a.num_pages) {
          phys = pg;
        } else if (a.status && report) {
          atomicOr(a.status, DEV_BAD_PAGE);
        }
      }
      for (int c = 0; c < D / 64; ++c) tma_load_4d(dst + c * L::kChunk + u * rows * 128, m, bar, c * 64, w.hk, slot, phys);
    }
  } else {
    (void)absent;
    (void)report;
    for (int c = 0; c < D / 64; ++c) tma_load_4d(dst + c * L::kChunk, m, bar, c * 64, t * kKeys, w.hk, w.b);
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
// Which column pairs take the FMA-pipe exponential: 3 of every 16. The MUFU
// pipe issues one ex2 per 8 cycles per warp; the polynomial costs a handful of
// packed FMA-pipe ops per pair, so moving a small share off MUFU balances the two pipes
// without starving the mask/max/convert work that also needs issue slots.
// (Measured on the softcap and ALiBi kernels too: all exponentials on MUFU
// was 1-2 % slower there.)
__device__ __forceinline__ constexpr bool exp_on_fma(int j) { return (j % 16) >= 13; }

// tanh on the FMA pipe for |y| <= kTanhPolyMax: the Taylor series
// y - y^3/3 + 2y^5/15 - 17y^7/315. The series alternates, so the error is
// below the first dropped term, 62y^9/2835 < 1.8e-6 there: after the cap
// (30 in the softcap workload) about 5e-5 on the score, far below the bf16
// rounding that P gets.
constexpr float kTanhPolyMax = 0.35f;
constexpr float kTanhA3 = -1.0f / 3.0f;
constexpr float kTanhA5 = 2.0f / 15.0f;
constexpr float kTanhA7 = -17.0f / 315.0f;

// Score mods for one 32-column chunk of a row (chunk index c), turning raw
// scores into log2-domain scores:
//   softcap: x = c*log2(e) * tanh(s*scale/c);  alibi: x = s*scale*log2(e) + slope*log2(e)*(kv - q_pos)
template <bool DECODE, int MOD>
__device__ __forceinline__ void mod_chunk(const FwdArgs& a, const Work& w, int s, int row, int t, int c, float* x,
                                          float off = 0.0f) {
  if constexpr (MOD == MOD_SOFTCAP) {
    const float k1 = a.softcap_k1;
    const float cl = a.softcap * kLog2e;
    float smax = 0.f;
#pragma unroll
    for (int i = 0; i < 32; i += 2) smax = max3(smax, fabsf(x[i]), fabsf(x[i + 1]));
    if (smax * k1 <= kTanhPolyMax) {
      // cl * tanh(k1 x) = x * (c0 + c1 z + c2 z^2 + c3 z^3) with z = x^2: the
      // series above with y = k1 x and the cap folded into the coefficients,
      // five packed ops per pair of scores.
      const float k1s = k1 * k1;
      const float c0 = cl * k1, c1 = c0 * kTanhA3 * k1s, c2 = c0 * kTanhA5 * (k1s * k1s),
                  c3 = c0 * kTanhA7 * (k1s * k1s * k1s);
      const float2 C0 = make_float2(c0, c0), C1 = make_float2(c1, c1), C2 = make_float2(c2, c2),
                   C3 = make_float2(c3, c3);
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        const float2 v = make_float2(x[i], x[i + 1]);
        const float2 z = mul2(v, v);
        float2 q = fma2(z, C3, C2);
        q = fma2(z, q, C1);
        q = fma2(z, q, C0);
        const float2 r = mul2(v, q);
        x[i] = r.x;
        x[i + 1] = r.y;
      }
    } else {
      // Some score of this chunk is large: tanh(y) = 1 - 2 / (e^{2y} + 1) on the SFU.
      const float k2 = 2.0f * k1 * kLog2e;
#pragma unroll
      for (int i = 0; i < 32; ++i) x[i] = cl * (1.0f - 2.0f * rcp(ex2(x[i] * k2) + 1.0f));
    }
  } else if constexpr (MOD == MOD_RELU) {
    // activation wrapper: the scaled score itself (the ReLU follows the mask)
    const float2 SC = make_float2(a.scale, a.scale);
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      const float2 r = mul2(make_float2(x[i], x[i + 1]), SC);
      x[i] = r.x;
      x[i + 1] = r.y;
    }
  } else if constexpr (MOD == MOD_ALIBI) {
    // decode rows sit at the last q_len positions of the sequence
    const long q_pos = DECODE ? (long)w.seqlen - a.q_len + min(row / a.g, a.q_len - 1)
                              : (long)(w_row0(w, s) + row) + a.q_offset;
    const int head = w_head(w, s) + (DECODE ? row % a.g : 0);
    const float slope = a.alibi[(int64_t)w.b * a.alibi_bstride + min(head, a.Hq - 1)] * kLog2e;
    // off (0, or minus the row's reference max) rides along with the bias
    const float base = slope * (float)((long)t * kKeys + 32 * c - q_pos) + off;
    const float2 SC = make_float2(a.scale_log2, a.scale_log2), SL = make_float2(slope, slope);
    const float2 B = make_float2(base, base);
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      const float2 bias = fma2(SL, make_float2((float)i, (float)(i + 1)), B);
      const float2 r = fma2(make_float2(x[i], x[i + 1]), SC, bias);
      x[i] = r.x;
      x[i + 1] = r.y;
    }
  }
}

// Per-row mask bounds of one partial tile, computed once per step. Column
// offset j (0..127) is allowed iff (unsigned)(j - clo) <= span, and for the
// document mask also doc[kv0 + j] == dq.
struct MaskRow {
  int clo;
  unsigned span;  // 0xffffffff sentinel handled by 'none'
  bool none;
  bool by_id;     // document mask with unsorted ids: compare ids per key
  int dq;         // document id of the query row (by_id)
  const int32_t* doc;  // document ids of this batch (by_id)
};

template <bool DECODE, bool BM>
__device__ __forceinline__ MaskRow mask_row(const FwdArgs& a, const Work& w, int s, int row, int t) {
  MaskRow m;
  const int kv0 = t * kKeys;
  long lo, hi;
  m.dq = 0;
  m.doc = a.doc_id;
  m.by_id = false;
  if constexpr (DECODE) {
    lo = 0;
    hi = (long)w.seqlen - 1 - (a.q_causal ? (long)(a.q_len - 1 - min(row / a.g, a.q_len - 1)) : 0l);
  } else {
    const int qrow = w_row0(w, s) + row;
    const long q_pos = (long)qrow + a.q_offset;
    if (BM && a.mask == MASK_DOCUMENT) {
      // Sorted ids: the row's keys are the interval [start of its run, q]
      // and take the range path; otherwise ids are compared key by key.
      const int bs = a.bm_Bm == 1 ? 0 : w.b;
      hi = q_pos;
      if (__ldg(a.bm_doc_sorted + bs)) {
        lo = __ldg(a.bm_doc_start + (int64_t)bs * a.Sq + min(qrow, a.Sq - 1));
      } else {
        lo = 0;
        m.by_id = true;
        m.doc = a.doc_id + (int64_t)w.b * a.doc_bstride;
        m.dq = m.doc[min(qrow, a.Sq - 1)];
      }
    } else {
      lo = a.wl >= 0 ? q_pos - a.wl : -(1l << 40);
      hi = a.wr >= 0 ? q_pos + a.wr : (1l << 40);
    }
    hi = min(hi, (long)a.Skv - 1);
  }
  const long clo = max(lo - kv0, 0l), chi = min(hi - kv0, (long)kKeys - 1);
  m.none = chi < clo;
  m.clo = (int)min(clo, (long)kKeys);
  m.span = m.none ? 0u : (unsigned)(chi - clo);
  return m;
}

// Applies the mask to chunk c (columns 32c .. 32c+31) of a partial tile. For
// the prefill window forms (causal included) the row's allowed range becomes
// a 32-bit mask for the chunk, so each element costs one bit test and one
// select; decode (only a split's ragged last tile) and the document mask keep
// the range compare, which needs fewer live registers. Without a block mask
// (BM false) a chunk allowed for the whole warp skips the selects, and the
// return value tells the caller that a chunk is masked for every row of the
// warp, so its exponentials are skipped (in block-mask kernels these votes
// cost more registers than they save).
template <bool DECODE, bool BM>
__device__ __forceinline__ bool mask_chunk(const FwdArgs& a, const MaskRow& m, int t, int c, float* x) {
  const float NEG_INF = -__int_as_float(0x7f800000);
  if (BM && a.mask == MASK_DOCUMENT && m.by_id) {
    const int kv = t * kKeys + 32 * c;
    const int4* d4 = reinterpret_cast<const int4*>(m.doc + kv);
    // keys of this chunk inside the sequence: whole groups of four are read
    // as one 16-byte load, a ragged last group (Skv not a multiple of 4)
    // element by element; keys past Skv fail the span test below anyway.
    const int nval = max(min(32, a.Skv - kv), 0);
    const int n4 = nval / 4, tail = nval % 4;
#pragma unroll
    for (int i4 = 0; i4 < 8; ++i4) {
      // volatile: keeps the load inside its chunk instead of letting all 32
      // of a tile be hoisted (and spilled) ahead of the loop
      int4 d = make_int4(-1, -1, -1, -1);
      if (i4 < n4) {
        asm volatile("ld.global.nc.v4.s32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(d.x), "=r"(d.y), "=r"(d.z), "=r"(d.w)
                     : "l"(d4 + i4));
      } else if (i4 == n4 && tail > 0) {
        const int32_t* dp = m.doc + kv + 4 * i4;
        d.x = __ldg(dp);
        if (tail > 1) d.y = __ldg(dp + 1);
        if (tail > 2) d.z = __ldg(dp + 2);
      }
      const int j = 32 * c + 4 * i4;
      x[4 * i4 + 0] = (!m.none && (unsigned)(j + 0 - m.clo) <= m.span && d.x == m.dq) ? x[4 * i4 + 0] : NEG_INF;
      x[4 * i4 + 1] = (!m.none && (unsigned)(j + 1 - m.clo) <= m.span && d.y == m.dq) ? x[4 * i4 + 1] : NEG_INF;
      x[4 * i4 + 2] = (!m.none && (unsigned)(j + 2 - m.clo) <= m.span && d.z == m.dq) ? x[4 * i4 + 2] : NEG_INF;
      x[4 * i4 + 3] = (!m.none && (unsigned)(j + 3 - m.clo) <= m.span && d.w == m.dq) ? x[4 * i4 + 3] : NEG_INF;
    }
    return false;
  } else if constexpr (DECODE) {
#pragma unroll
    for (int i = 0; i < 32; ++i) x[i] = (!m.none && (unsigned)(32 * c + i - m.clo) <= m.span) ? x[i] : NEG_INF;
    return false;
  } else {
    const int lo = m.clo - 32 * c, hi = m.clo + (int)m.span - 32 * c;
    unsigned bits = 0u;
    if (!m.none && hi >= 0 && lo <= 31) bits = (0xffffffffu >> (31 - min(hi, 31))) & (0xffffffffu << max(lo, 0));
    if (!BM && __all_sync(0xffffffffu, bits == 0xffffffffu)) return false;
    const bool dead = !BM && __all_sync(0xffffffffu, bits == 0u);
#pragma unroll
    for (int i = 0; i < 32; ++i) x[i] = (bits & (1u << i)) ? x[i] : NEG_INF;
    return dead;
  }
}

// Exponentials of one 32-column chunk (16 pairs) against reference max -nmu,
// packed to bf16 pairs; sums and the chunk max are accumulated on the way.
// AFFINE false: x already holds the exponents (MULT and NMU unused).
template <bool AFFINE = true>
__device__ __forceinline__ void exp_chunk(const float* x, float2 MULT, float2 NMU, uint32_t* pk, float2& acc0,
                                          float2& acc1) {
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const float2 arg = AFFINE ? fma2(make_float2(x[2 * j], x[2 * j + 1]), MULT, NMU)
                              : make_float2(x[2 * j], x[2 * j + 1]);
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

// Streams one tile out of TMEM 32 columns at a time: mods, mask (MASKED),
// optimistic exponentials, P chunk stores. Returns the raw row max.
// With 'guess' set (the row has no reference max yet), the reference is taken
// from chunk 0 of this tile and returned through ref_out (log2 units).
template <bool DECODE, int MOD, bool MASKED, bool BM>
__device__ __forceinline__ float stream_tile(const FwdArgs& a, const Work& w, int s, int row, int t, uint32_t tS,
                                             float* x, float nmu0, float2& acc0, float2& acc1, bool guess,
                                             float& ref_out) {
  const float NEG_INF = -__int_as_float(0x7f800000);
  const float mult = MOD == MOD_NONE ? a.scale_log2 : 1.0f;
  const float2 MULT = make_float2(mult, mult);
  float2 NMU = make_float2(nmu0, nmu0);
  MaskRow mr;
  if constexpr (MASKED) mr = mask_row<DECODE, BM>(a, w, s, row, t);
  float mc = NEG_INF;
  // All four chunks are requested before a single wait: one exposed TMEM
  // load latency per tile instead of one per chunk (measured 2.5 % faster
  // on the causal prefill than keeping one chunk in flight).
#pragma unroll
  for (int c = 0; c < 4; ++c) tmem_ld32f(tS + 32 * c, x + 32 * c);
  tmem_ld_wait();
  reg_fence_f<128>(x);
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    if constexpr (MOD != MOD_NONE) mod_chunk<DECODE, MOD>(a, w, s, row, t, c, x + 32 * c);
    bool dead = false;
    if constexpr (MASKED) dead = mask_chunk<DECODE, BM>(a, mr, t, c, x + 32 * c);
    mc = fmaxf(mc, chunk_max(x + 32 * c));
    if (c == 0 && guess) {
      const float g = mc * mult;
      ref_out = g;
      NMU = make_float2(g == NEG_INF ? 0.0f : -g, g == NEG_INF ? 0.0f : -g);
    }
    uint32_t pk[16];
    if (MASKED && !BM && dead) {
      // every score of this chunk is masked for the whole warp: P = 0
#pragma unroll
      for (int j = 0; j < 16; ++j) pk[j] = 0u;
    } else {
      exp_chunk(x + 32 * c, MULT, NMU, pk, acc0, acc1);
    }
    tmem_st16(tS + 16 * c, pk);
  }
  return mc;
}

// Scores of a whole tile with mods and mask (all four chunks requested from
// TMEM before one wait); returns the row max of the modded scores. The
// exponentials follow once the reference is known. off is added to the ALiBi
// bias (minus the row's reference max in prefill, else 0).
template <bool DECODE, int MOD, bool MASKED, bool BM>
__device__ __forceinline__ float prepare_tile(const FwdArgs& a, const Work& w, int s, int row, int t, uint32_t tS,
                                              float* x, float off = 0.0f) {
  const float NEG_INF = -__int_as_float(0x7f800000);
  MaskRow mr;
  if constexpr (MASKED) mr = mask_row<DECODE, BM>(a, w, s, row, t);
  float mc = NEG_INF;
#pragma unroll
  for (int c = 0; c < 4; ++c) tmem_ld32f(tS + 32 * c, x + 32 * c);
  tmem_ld_wait();
  reg_fence_f<128>(x);
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    if constexpr (MOD != MOD_NONE) mod_chunk<DECODE, MOD>(a, w, s, row, t, c, x + 32 * c, off);
    if constexpr (MASKED) (void)mask_chunk<DECODE, BM>(a, mr, t, c, x + 32 * c);
    mc = fmaxf(mc, chunk_max(x + 32 * c));
  }
  return mc;
}

// One key tile of the online softmax for one query row (this thread's TMEM
// lane). The exponentials are taken optimistically against the row's current
// reference max while the scores stream in from TMEM chunk by chunk; only if
// some row of the warp finds a max more than 8 above its reference (always on
// the first tile) is the tile redone against the new max, with O rescaled.
template <int D, bool DECODE, int MOD, bool BM>
__device__ __forceinline__ void softmax_step(const FwdArgs& a, const Work& w, int s, int row, int t, int cls,
                                             uint32_t tS, uint32_t tO, bool first, RowState& st,
                                             uint64_t* p_ready) {
  float x[kKeys];
  const float NEG_INF = -__int_as_float(0x7f800000);
  if constexpr (MOD == MOD_RELU) {
    // Activation wrapper (the FlexAttention talk's ReLU example): P = max(scale
    // * s, 0) on allowed pairs, no running max, no rescale, no normalisation.
    // The row keeps m = 0 and l = the summed weights, so the epilogue writes
    // ln(l) in the LSE slot and O unscaled.
    float wsum = 0.f;
    if (cls == 0) {
      uint32_t pk[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) pk[j] = 0u;
      tmem_st32(tS, pk);
      tmem_st32(tS + 32, pk);
    } else {
      if (cls == 2)
        (void)prepare_tile<DECODE, MOD, false, BM>(a, w, s, row, t, tS, x);
      else
        (void)prepare_tile<DECODE, MOD, true, BM>(a, w, s, row, t, tS, x);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float p0 = fmaxf(x[32 * c + 2 * j], 0.f), p1 = fmaxf(x[32 * c + 2 * j + 1], 0.f);
          wsum += p0 + p1;
          pk[j] = pack_bf16x2(p0, p1);
        }
        tmem_st16(tS + 16 * c, pk);
      }
    }
    tmem_st_wait();
    tc_fence_before();
    mbar_arrive(p_ready);
    st.m = 0.f;
    st.l += wsum;
    (void)tO;
    (void)first;
    return;
  }
  const float mult = MOD == MOD_NONE ? a.scale_log2 : 1.0f;  // x * mult is the log2-domain score
  const float2 MULT = make_float2(mult, mult);
  float2 acc0 = make_float2(0.f, 0.f), acc1 = acc0;
  float mt;
  const bool have_ref = !first && __all_sync(0xffffffffu, st.m != NEG_INF);
  const float nmu0 = have_ref ? -st.m : 0.0f;
  float xref = 0.0f;  // the scores in x are relative to this (prefill ALiBi with a reference max)
  bool guessed = false;
  if (cls == 0) {
#pragma unroll
    for (int c = 0; c < kKeys; ++c) x[c] = NEG_INF;
    mt = NEG_INF;
    uint32_t pk[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) pk[j] = 0u;
    tmem_st32(tS, pk);
    tmem_st32(tS + 32, pk);
  } else if (MOD == MOD_NONE) {
    // Streamed: chunk c+1 is in flight while chunk c is (masked and)
    // exponentiated against the row's reference max; a row without one yet
    // (first tile, or only masked keys so far) takes the max of its first
    // chunk instead, corrected below if the tile exceeds it by more than the
    // threshold. Full and partial tiles run separate instantiations so the
    // common one stays compact.
    const bool my_guess = first || st.m == NEG_INF;
    float guess_ref = NEG_INF;
    const float my_nmu = my_guess ? 0.0f : -st.m;
    if (cls == 2)
      mt = stream_tile<DECODE, MOD, false, BM>(a, w, s, row, t, tS, x, my_nmu, acc0, acc1, my_guess, guess_ref) * mult;
    else
      mt = stream_tile<DECODE, MOD, true, BM>(a, w, s, row, t, tS, x, my_nmu, acc0, acc1, my_guess, guess_ref) * mult;
    if (my_guess) {
      // This row's exponentials are relative to the guess, which becomes its
      // reference; its l and O are still empty (or all zero).
      st.m = guess_ref;
      st.l = 0.0f;
    }
    guessed = true;
  } else {
    // Scores (with mods and mask) first; the exponentials follow against the
    // reference max when there is one, else in the slow path below. With
    // ALiBi in prefill the reference rides in the bias (x relative to xref).
    constexpr bool kFold = kFoldRef<MOD> && !DECODE;
    const float off = (kFold && have_ref) ? -st.m : 0.0f;
    xref = -off;
    float mc;
    if (cls == 2)
      mc = prepare_tile<DECODE, MOD, false, BM>(a, w, s, row, t, tS, x, off);
    else
      mc = prepare_tile<DECODE, MOD, true, BM>(a, w, s, row, t, tS, x, off);
    mt = mc * mult + xref;
    if (have_ref) {
      const float2 NMU = make_float2(nmu0, nmu0);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
        if constexpr (kFold)
          exp_chunk<false>(x + 32 * c, MULT, NMU, pk, acc0, acc1);
        else
          exp_chunk(x + 32 * c, MULT, NMU, pk, acc0, acc1);
        tmem_st16(tS + 16 * c, pk);
      }
    }
  }
  // Slow path: no reference max yet (and none guessed), or a max that grew
  // past the threshold.
  const bool grow = (!have_ref && !guessed) || mt > st.m + kRescaleThreshold;
  float alpha = 1.0f;
  if (__any_sync(0xffffffffu, grow) && cls != 0) {
    const float m_new = fmaxf(st.m, mt);
    alpha = (m_new == NEG_INF || st.m == NEG_INF) ? (st.m == NEG_INF ? 0.0f : 1.0f) : ex2(st.m - m_new);
    st.m = m_new;
    const float nmu = (m_new == NEG_INF) ? 0.0f : (kFoldRef<MOD> && !DECODE ? xref - m_new : -m_new);
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

// ---------------------------------------------------------------- prefill, half tiles
// The softcap kernel hands each key tile to the tensor pipe in two halves:
// its softmax (tanh series, then exponentials) is long enough that
// overlapping it with the MMAs pays for the extra hand-offs (whole tiles
// measured 11 % slower). Without a mod, and with ALiBi since its tiles are
// walked from the diagonal back (no rescales), whole tiles are faster (the
// half schedule measured 5 % and 7 % slower).
template <bool DECODE, int MOD>
constexpr bool kHalfTiles = !DECODE && MOD == MOD_SOFTCAP;

// With half tiles: P for keys
// 0-63 goes to S(s) columns [0, 32) and P for keys 64-127 to [64, 96), so:
//   - once P of keys 0-63 is written, PV over those keys and the next tile's
//     QK^T for keys 0-63 (into columns [0, 64)) run while the softmax works on
//     keys 64-127;
//   - once P of keys 64-127 is written, PV over them and the next tile's
//     QK^T for keys 64-127 (into [64, 128)) follow.
// The softmax of the next tile starts on its first half while the tensor
// pipe finishes the second, so neither waits for the other's whole tile.

// Half h of a key tile (chunks 2h, 2h+1: S(s) columns [64h, 64h+64)),
// streamed like stream_tile: chunk 2h+1 is in flight while chunk 2h is
// exponentiated. x holds the half's 64 scores.
template <int MOD, bool MASKED, bool BM>
__device__ __forceinline__ float stream_half(const FwdArgs& a, const Work& w, int s, int row, int t, uint32_t tS,
                                             int h, float* x, float nmu0, float2& acc0, float2& acc1, bool guess,
                                             float& ref_out) {
  const float NEG_INF = -__int_as_float(0x7f800000);
  const float mult = MOD == MOD_NONE ? a.scale_log2 : 1.0f;
  const float2 MULT = make_float2(mult, mult);
  float2 NMU = make_float2(nmu0, nmu0);
  MaskRow mr;
  if constexpr (MASKED) mr = mask_row<false, BM>(a, w, s, row, t);
  float mc = NEG_INF;
  const uint32_t base = tS + 64 * h;
  tmem_ld32f(base, x);
  tmem_ld32f(base + 32, x + 32);
  tmem_ld_wait();
  reg_fence_f<64>(x);
#pragma unroll
  for (int cc = 0; cc < 2; ++cc) {
    const int c = 2 * h + cc;
    if constexpr (MOD != MOD_NONE) mod_chunk<false, MOD>(a, w, s, row, t, c, x + 32 * cc);
    bool dead = false;
    if constexpr (MASKED) dead = mask_chunk<false, BM>(a, mr, t, c, x + 32 * cc);
    mc = fmaxf(mc, chunk_max(x + 32 * cc));
    if (cc == 0 && guess) {
      const float g = mc * mult;
      ref_out = g;
      NMU = make_float2(g == NEG_INF ? 0.0f : -g, g == NEG_INF ? 0.0f : -g);
    }
    uint32_t pk[16];
    if (MASKED && !BM && dead) {
#pragma unroll
      for (int j = 0; j < 16; ++j) pk[j] = 0u;
    } else {
      exp_chunk(x + 32 * cc, MULT, NMU, pk, acc0, acc1);
    }
    tmem_st16(base + 16 * cc, pk);
  }
  return mc;
}

// Half h with score mods: the half's scores (mods, mask) first, then its
// exponentials once the reference is known.
template <int MOD, bool MASKED, bool BM>
__device__ __forceinline__ float prepare_half(const FwdArgs& a, const Work& w, int s, int row, int t, uint32_t tS,
                                              int h, float* x) {
  const float NEG_INF = -__int_as_float(0x7f800000);
  MaskRow mr;
  if constexpr (MASKED) mr = mask_row<false, BM>(a, w, s, row, t);
  float mc = NEG_INF;
  const uint32_t base = tS + 64 * h;
  tmem_ld32f(base, x);
  tmem_ld32f(base + 32, x + 32);
  tmem_ld_wait();
  reg_fence_f<64>(x);
#pragma unroll
  for (int cc = 0; cc < 2; ++cc) {
    const int c = 2 * h + cc;
    if constexpr (MOD != MOD_NONE) mod_chunk<false, MOD>(a, w, s, row, t, c, x + 32 * cc);
    if constexpr (MASKED) (void)mask_chunk<false, BM>(a, mr, t, c, x + 32 * cc);
    mc = fmaxf(mc, chunk_max(x + 32 * cc));
  }
  return mc;
}

// Multiplies this row's O accumulator by alpha in TMEM.
template <int D>
__device__ __forceinline__ void rescale_o(uint32_t tO, float alpha) {
#pragma unroll 1
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

// One key tile of the prefill online softmax for one query row, as two
// halves. The exponentials of a half are taken against the row's reference
// max (the first chunk's max when the row has none yet); when some row of
// the warp finds the half's max more than 8 above its reference, the half is
// redone against the new max and O is rescaled, after waiting for the PVs
// that may still be adding into O: for the first half, the previous tile's
// second-half PV (done once this tile's keys 64-127 are in S); for the second
// half, this tile's first-half PV. On entry S of keys 0-63 is ready. g is the
// step's barrier phase index; returns false if a wait gave up.
template <int D, int MOD, bool BM>
__device__ __forceinline__ bool softmax_step_halves(const FwdArgs& a, const Work& w, int s, int row, int t, int cls,
                                                    uint32_t tS, uint32_t tO, bool first, RowState& st, Barriers& bar,
                                                    int g, volatile int* abort_flag) {
  const float NEG_INF = -__int_as_float(0x7f800000);
  const float mult = MOD == MOD_NONE ? a.scale_log2 : 1.0f;
  const float2 MULT = make_float2(mult, mult);
  const uint32_t par = (uint32_t)(g & 1);
  bool b_ready = false;  // S of keys 64-127 already waited for
#pragma unroll 1
  for (int h = 0; h < 2; ++h) {
    if (h == 1 && !b_ready) {
      ATTN_TRACE_REC(threadIdx.x / 32, EV_SB_WAIT, g);
      if (!__all_sync(0xffffffffu, mbar_wait_spin(&bar.s_b_ready[s], par, abort_flag))) return false;
      tc_fence_after();
      ATTN_TRACE_REC(threadIdx.x / 32, EV_SB_READY, g);
    }
    float x[64];
    float2 acc0 = make_float2(0.f, 0.f), acc1 = acc0;
    float mh;
    const bool have_ref = __all_sync(0xffffffffu, st.m != NEG_INF);
    bool guessed = false;
    if (cls == 0) {
#pragma unroll
      for (int c = 0; c < 64; ++c) x[c] = NEG_INF;
      mh = NEG_INF;
      uint32_t pk[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) pk[j] = 0u;
      tmem_st32(tS + 64 * h, pk);
      guessed = true;
    } else if (MOD == MOD_NONE) {
      const bool my_guess = st.m == NEG_INF;
      float guess_ref = NEG_INF;
      const float my_nmu = my_guess ? 0.0f : -st.m;
      if (cls == 2)
        mh = stream_half<MOD, false, BM>(a, w, s, row, t, tS, h, x, my_nmu, acc0, acc1, my_guess, guess_ref) * mult;
      else
        mh = stream_half<MOD, true, BM>(a, w, s, row, t, tS, h, x, my_nmu, acc0, acc1, my_guess, guess_ref) * mult;
      if (my_guess) {
        // the guess becomes this row's reference; its l and O hold nothing yet
        st.m = guess_ref;
        st.l = 0.0f;
      }
      guessed = true;
    } else {
      float mc;
      if (cls == 2)
        mc = prepare_half<MOD, false, BM>(a, w, s, row, t, tS, h, x);
      else
        mc = prepare_half<MOD, true, BM>(a, w, s, row, t, tS, h, x);
      mh = mc * mult;
      if (have_ref) {
        const float2 NMU = make_float2(-st.m, -st.m);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t pk[16];
          exp_chunk(x + 32 * c, MULT, NMU, pk, acc0, acc1);
          tmem_st16(tS + 64 * h + 16 * c, pk);
        }
      }
    }
    const bool grow = (!have_ref && !guessed) || mh > st.m + kRescaleThreshold;
    float alpha = 1.0f;
    if (__any_sync(0xffffffffu, grow) && cls != 0) {
      const float m_new = fmaxf(st.m, mh);
      alpha = (m_new == NEG_INF || st.m == NEG_INF) ? (st.m == NEG_INF ? 0.0f : 1.0f) : ex2(st.m - m_new);
      st.m = m_new;
      const float nmu = (m_new == NEG_INF) ? 0.0f : -m_new;
      const float2 NMU = make_float2(nmu, nmu);
      acc0 = acc1 = make_float2(0.f, 0.f);
      tmem_st_wait();  // the optimistic P stores land before they are overwritten
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t pk[16];
        exp_chunk(x + 32 * c, MULT, NMU, pk, acc0, acc1);
        tmem_st16(tS + 64 * h + 16 * c, pk);
      }
      // O may still receive a PV: wait until it has landed, then rescale.
      bool have_o = true;
      if (h == 0) {
        // The first half's PV of this tile is not issued yet; the previous
        // tile's second-half PV completed before this tile's keys 64-127
        // were committed to S. At a unit's first tile O holds nothing.
        have_o = !first;
        if (have_o) {
          if (!__all_sync(0xffffffffu, mbar_wait_spin(&bar.s_b_ready[s], par, abort_flag))) return false;
          b_ready = true;
        }
      } else {
        if (!__all_sync(0xffffffffu, mbar_wait_spin(&bar.pv_a_done[s], par, abort_flag))) return false;
      }
      if (have_o) {
        tc_fence_after();
        rescale_o<D>(tO, alpha);
      }
    }
    tmem_st_wait();
    tc_fence_before();
    mbar_arrive(h == 0 ? &bar.p_ready[s] : &bar.p_b_ready[s]);
    if (h == 0) ATTN_TRACE_REC(threadIdx.x / 32, EV_HALF_A_DONE, g);
    acc0 = add2(acc0, acc1);
    st.l = st.l * alpha + (acc0.x + acc0.y);
  }
  return true;
}

// ---------------------------------------------------------------- kernel
// Epilogue of one unit for softmax subtile s: O / l to bf16 (prefill) or the
// merged, normalised split partial (decode), and the LSE.
template <int D, bool DECODE>
__device__ __forceinline__ bool epilogue(const FwdArgs& a, const CUtensorMap* map_o, const Work& w, int s, int row,
                                         uint32_t lane_base, bool have_o, const RowState& st, uint8_t* extra,
                                         Barriers& bar, int mcnt, volatile int* abort_flag) {
  using L = Layout<D, DECODE>;
  const float NEG_INF = -__int_as_float(0x7f800000);
  const uint32_t tO = lane_base + 256 + s * L::kOCols;
  if constexpr (!DECODE) {
    // Each warp writes its 32 rows as 64-column boxes: registers -> its SW128
    // staging box in shared memory -> one TMA store per box, so the global
    // writes are whole 128-byte lines instead of one row per lane.
    const int wq = row / 32, lane = row % 32;
    const int r0 = w_row0(w, s);
    const int h = w_head(w, s);
    const int qrow = r0 + row;
    const bool valid = qrow < a.Sq && r0 < a.Sq;
    const bool box_valid = r0 + 32 * wq < a.Sq;  // warp-uniform; rows past Sq are clipped by the map
    // the ReLU activation wrapper leaves O unnormalised
    const float inv_l = a.mod == MOD_RELU ? 1.0f : (st.l > 0.f ? 1.0f / st.l : 0.f);
    uint8_t* stage = extra + (s * 4 + wq) * L::kStageWarpBytes;
    const uint32_t srow = smem_u32(stage) + lane * 128;
#pragma unroll
    for (int hh = 0; hh < D / 64; ++hh) {
      float o[64];
      if (have_o) {
        tmem_ld64f(tO + 64 * hh, o);
        tmem_ld_wait();
        reg_fence_f<64>(o);
      } else {
#pragma unroll
        for (int j2 = 0; j2 < 64; ++j2) o[j2] = 0.f;
      }
      uint32_t pk[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) pk[e] = pack_bf16x2(o[2 * e] * inv_l, o[2 * e + 1] * inv_l);
      // The staging box is free once this warp's previous store has read it.
      if (lane == 0) bulk_wait_read_all();
      __syncwarp();
#pragma unroll
      for (int j = 0; j < 8; ++j)
        st_shared_v4(srow + ((uint32_t)(j ^ (lane & 7)) << 4), pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && box_valid) {
        tma_store_4d(map_o, stage, 64 * hh, r0 + 32 * wq, h, w.b);
        bulk_commit_group();
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
    float* merge_m = reinterpret_cast<float*>(extra);
    float* merge_l = merge_m + 128;
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
      const int h = w.head0 + row % a.g;
      const int ti = row / a.g;  // new token of the row
      const bool valid = row < a.g * a.q_len;
      const int64_t prow = (((int64_t)w.b * a.q_len + ti) * a.Hq + h) * a.n_splits + w.split;
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
//   k_full / v_full / k_empty / v_empty   once per K/V load.
// While the softmax warps write a unit's outputs, the producer already loads
// the next unit's Q and K/V and the MMA warp runs its first QK^T products.
template <int D, bool DECODE, int MOD, bool BM>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                    const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_o,
                    const FwdArgs a) {
  using L = Layout<D, DECODE>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Barriers& bar = *reinterpret_cast<Barriers*>(smem + L::kBarOff);
  uint8_t* extra = smem + L::kExtraOff;
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  volatile int* abort_flag = &bar.abort_flag;

  if (threadIdx.x == 0) {
    bar.abort_flag = 0;
#ifdef ATTN_TRACE
    bar.trace_t0 = clock64();
    for (int r = 0; r < kTraceRoles; ++r) bar.trace_cnt[r] = 0;
#endif
    mbar_init(&bar.q_full, 1);
    mbar_init(&bar.q_empty, 2);  // the last QK^T of each subtile's MMA warp
    for (int i = 0; i < L::kNSlot; ++i) {
      mbar_init(&bar.k_full[i], 1);
      mbar_init(&bar.v_full[i], 1);
      // prefill: both subtiles read every K/V tile; decode: one subtile does
      mbar_init(&bar.k_empty[i], DECODE ? 1 : 2);
      mbar_init(&bar.v_empty[i], DECODE ? 1 : 2);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar.s_ready[s], 1);
      mbar_init(&bar.p_ready[s], 128);
      mbar_init(&bar.s_b_ready[s], 1);
      mbar_init(&bar.p_b_ready[s], 128);
      mbar_init(&bar.pv_a_done[s], 1);
      mbar_init(&bar.o_done[s], 1);
      mbar_init(&bar.o_free[s], 128);
    }
    mbar_init(&bar.merge_full, 128);
    mbar_init(&bar.merge_empty, 128);
    mbar_init(&bar.final_mma[0], 1);
    mbar_init(&bar.final_mma[1], 1);
    mbar_init(&bar.mma_turn[0], 1);
    mbar_init(&bar.mma_turn[1], 1);
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
  // Polling variant for the per-step S-ready / P-ready hand-offs.
  auto wait_spin_all = [&](uint64_t* b, uint32_t par) {
    const bool got = mbar_wait_spin(b, par, abort_flag);
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
    int kload = 0;  // K/V tile pairs started so far: ring position and phase
    int vload = 0;  // V tiles issued so far (one behind kload while a pair is half issued)
    int qcnt = 0;   // units with key tiles so far
    bool ok = true;
    for (int r = 0; ok && r < rounds; ++r) {
      const int u = unit_of(r);
      if (u < 0) continue;
      const Work w = map_work<DECODE>(a, u);
      if constexpr (DECODE) {
        // one report per sequence: a length outside [0, max_seqlen]
        const int raw = a.seqlens[w.b];
        if (w.split == 0 && w.hk == 0 && (raw < 0 || raw > a.max_seqlen) && a.status && elect_one_sync())
          atomicOr(a.status, DEV_BAD_LEN);
        __syncwarp();
      }
      if constexpr (BM) {
        // caller-written tables: an order entry outside the q-tiles, or a
        // count outside [0, n_kv_tiles], is reported (and was not followed)
        const int qi = u / (a.B * (a.pair_heads ? a.Hq / 2 : a.Hq));
        bool bad = false;
        if (a.bm_row_order != nullptr && a.pair_heads) {
          const int o = __ldg(a.bm_row_order + (int64_t)(a.bm_Bm == 1 ? 0 : w.b) * a.bm_nQ + qi / (a.bm_rows / kRows));
          bad = o < 0 || o >= a.bm_nQ;
        }
        for (int s = 0; s < 2; ++s) {
          if (w_row0(w, s) >= a.Sq) continue;
          const int64_t q = bm_slice(a, w.b, w_head(w, s)) * a.bm_nQ + w_row0(w, s) / a.bm_rows;
          const int pc = __ldg(a.bm_part_cnt + q), fc = __ldg(a.bm_full_cnt + q);
          bad |= pc < 0 || pc > a.nK || fc < 0 || fc > a.nK;
        }
        if (bad && a.status && elect_one_sync()) atomicOr(a.status, DEV_BAD_MASK);
        __syncwarp();
      }
      TileWalker tw;
      const int n = walker_init<DECODE, BM, kDescWalk<DECODE, MOD>>(a, w, tw);
      if (n == 0) continue;
      if (qcnt > 0 && !wait_all(&bar.q_empty, (qcnt - 1) & 1)) {
        ok = false;
        break;
      }
      ATTN_TRACE_REC(TR_TMA, EV_Q_LOAD, qcnt);
      if (elect_one_sync()) {
        mbar_arrive_expect_tx(&bar.q_full, DECODE ? (uint32_t)a.q_bytes : (uint32_t)(L::kNQ * L::kTileBytes));
        for (int s = 0; s < L::kNQ; ++s)
          for (int c = 0; c < D / 64; ++c) {
            uint8_t* dst = smem + L::kQOff + s * L::kTileBytes + c * L::kChunk;
            if constexpr (DECODE) {
              // several new tokens: a (64, g, 1, tokens) box puts token i's
              // heads at rows i*g .. i*g + g - 1
              if (a.q_len > 1)
                tma_load_5d(dst, &map_q, &bar.q_full, c * 64, 0, w.hk, 0, w.b);
              else
                tma_load_3d(dst, &map_q, &bar.q_full, c * 64, w.head0, w.b);
            } else
              tma_load_4d(dst, &map_q, &bar.q_full, c * 64, w_row0(w, s), w_head(w, s), w.b);
          }
      }
      __syncwarp();
      if constexpr (!DECODE) {
        // Q is read once per unit, so the next unit's Q would come from HBM
        // while its first QK^T waits: pull it into L2 now, a unit ahead.
        const int un = r + 1 < rounds ? unit_of(r + 1) : -1;
        if (un >= 0) {
          const Work wn = map_work<DECODE>(a, un);
          if (elect_one_sync()) {
            for (int s = 0; s < 2; ++s)
              if (w_row0(wn, s) < a.Sq)
                for (int c = 0; c < D / 64; ++c) tma_prefetch_l2_4d(&map_q, c * 64, w_row0(wn, s), w_head(wn, s), wn.b);
          }
          __syncwarp();
        }
      }
      ++qcnt;
      const int n_loads = DECODE ? 2 * n : n;
      for (int k = 0; k < n_loads; ++k) {
        const int t = tw.t;
        const int slot = kload % L::kNSlot;
        const int use = kload / L::kNSlot;
        const bool absent = DECODE && t >= w.t_end;
        // K and V of a slot are released separately (K once its last QK^T has
        // read it, V after its last PV), so the next K can land a step earlier.
        if (use > 0 && !wait_all(&bar.k_empty[slot], (use - 1) & 1)) {
          ok = false;
          break;
        }
        ATTN_TRACE_REC(TR_TMA, EV_KV_LOAD, kload);
        if (elect_one_sync())
          load_kv_tile<D, DECODE>(a, w, &map_k, smem + L::kKOff + slot * L::kTileBytes, &bar.k_full[slot], t, absent,
                                  true);
        __syncwarp();
        ++kload;
        if (use > 0 && !wait_all(&bar.v_empty[slot], (use - 1) & 1)) {
          ok = false;
          break;
        }
        if (elect_one_sync())
          load_kv_tile<D, DECODE>(a, w, &map_v, smem + L::kVOff + slot * L::kTileBytes, &bar.v_full[slot], t, absent,
                                  false);
        __syncwarp();
        ++vload;
        if (DECODE)
          ++tw.t;
        else
          walker_next<BM, kDescWalk<DECODE, MOD>>(tw);
      }
    }
    // Drain: on an abort, wait (bounded) for every copy still in flight so
    // none lands in shared memory after the CTA has exited.
    if (*abort_flag) {
      for (int k = max(0, kload - L::kNSlot); k < kload; ++k)
        mbar_wait_timeout(&bar.k_full[k % L::kNSlot], (k / L::kNSlot) & 1);
      for (int k = max(0, vload - L::kNSlot); k < vload; ++k)
        mbar_wait_timeout(&bar.v_full[k % L::kNSlot], (k / L::kNSlot) & 1);
      if (qcnt > 0) mbar_wait_timeout(&bar.q_full, (qcnt - 1) & 1);
    }
  } else if (warp == kMmaWarp || (kMmaWarps == 2 && warp == kMmaWarp1)) {
    regs_decrease<kControlRegs>();
    // ------------------------------------------------------------ MMA issue
    // A thread that issues tcgen05.mma stalls until the tensor pipe accepts
    // the MMA, so every wait and fence between two batches of MMAs leaves the
    // pipe idle: a step's PV and the next QK^T of a subtile therefore go out
    // back to back from one elected lane. The subtiles take turns in a fixed
    // order (PV(0) QK(0) PV(1) QK(1) per step), which keeps the ping-pong:
    // one subtile's softmax runs while the other's MMAs execute.
    // With kMmaWarps == 2 each subtile has its own issuing warp and the two
    // hand a turn token to each other, so one warp's waits overlap the other
    // warp's batch.
    constexpr int kSubPerWarp = kMmaWarps == 2 ? 1 : 2;
    const int s_first = (kMmaWarps == 2 && warp == kMmaWarp1) ? 1 : 0;
    const int trole = warp;
    (void)trole;
    constexpr uint32_t idesc_qk = idesc_bf16_f32(128, kKeys, 0, 0);
    constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
    // Descriptor low words (start address in 16-byte units + LBO); every
    // per-MMA offset below is a compile-time constant added to them.
    constexpr uint32_t kHi = sdesc_sw128_hi(1024);
    const uint32_t q_lo = sdesc_sw128_lo(smem_u32(smem + L::kQOff), 16);
    const uint32_t k_lo = sdesc_sw128_lo(smem_u32(smem + L::kKOff), 16);
    const uint32_t v_lo = sdesc_sw128_lo(smem_u32(smem + L::kVOff), L::kChunk);
    constexpr uint32_t kTileUnits = L::kTileBytes >> 4;
    // QK^T of subtile s into S(s) (elected lane only). last: the unit's
    // final QK^T of s, after which (once both subtiles' are done) Q may be
    // reloaded. The K tile of the slot is released once every subtile that
    // reads it has issued its QK^T.
    auto qk_mmas = [&](int s, int slot, bool last) {
      const uint32_t qa = q_lo + (DECODE ? 0u : (uint32_t)s * kTileUnits);
      const uint32_t ka = k_lo + (uint32_t)slot * kTileUnits;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = ((kk / 4) * L::kChunk + (kk % 4) * 32) >> 4;
        mma_ss(tmem + s * 128, sdesc_join(qa + off, kHi), sdesc_join(ka + off, kHi), idesc_qk, kk > 0);
      }
      mma_commit(&bar.s_ready[s]);
      if (last) mma_commit(&bar.q_empty);
      mma_commit(&bar.k_empty[slot]);
    };
    // Prefill with the softcap: QK^T and PV in key halves (see "prefill, half tiles").
    constexpr uint32_t idesc_qk_half = idesc_bf16_f32(128, 64, 0, 0);
    constexpr uint32_t kHalfKeyUnits = (64 * 128) >> 4;  // 64 K rows of a 128-byte SW128 box
    auto qk_half_mmas = [&](int s, int slot, int h, bool last) {
      const uint32_t qa = q_lo + (uint32_t)s * kTileUnits;
      const uint32_t ka = k_lo + (uint32_t)slot * kTileUnits + (uint32_t)h * kHalfKeyUnits;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = ((kk / 4) * L::kChunk + (kk % 4) * 32) >> 4;
        mma_ss(tmem + s * 128 + 64 * h, sdesc_join(qa + off, kHi), sdesc_join(ka + off, kHi), idesc_qk_half, kk > 0);
      }
      mma_commit(h == 0 ? &bar.s_ready[s] : &bar.s_b_ready[s]);
      if (last) mma_commit(&bar.q_empty);
      if (h == 1) mma_commit(&bar.k_empty[slot]);
    };
    auto slot_of = [&](int g, int s) { return DECODE ? (2 * g + s) % L::kNSlot : g % L::kNSlot; };
    auto phase_of = [&](int g, int s) { return (uint32_t)(((DECODE ? 2 * g + s : g) / L::kNSlot) & 1); };
    // Steps of round r's unit (0 if it has none). The MMA warp needs nothing
    // else about a unit. The next round's count is taken right after a
    // unit's first QK^T products are issued, while the softmax works on
    // them: this once-per-unit code has usually left the instruction cache,
    // and its refetch is hidden there instead of delaying the next QK^T.
    auto unit_steps = [&](int r) -> int {
      const int u = r < rounds ? unit_of(r) : -1;
      if (u < 0) return 0;
      const Work w = map_work<DECODE>(a, u);
      TileWalker tw;
      return walker_init<DECODE, BM, kDescWalk<DECODE, MOD>>(a, w, tw);
    };
    // Turn token between two issuing warps: batch b of subtile 1 follows
    // batch b of subtile 0, batch b + 1 of subtile 0 follows batch b of
    // subtile 1 (one arrival each; phases count batches).
    int batch = 0;
    auto take_turn = [&](int s) -> bool {
      if constexpr (kMmaWarps == 2) {
        if (s == 1) return wait_spin_all(&bar.mma_turn[1], batch & 1);
        if (batch > 0) return wait_spin_all(&bar.mma_turn[0], (batch - 1) & 1);
      }
      (void)s;
      return true;
    };
    auto pass_turn = [&](int s) {
      if constexpr (kMmaWarps == 2) {
        if (elect_one_sync()) mbar_arrive(&bar.mma_turn[s ^ 1]);
        __syncwarp();
      }
      (void)s;
    };
    int gstep = 0;  // steps issued so far across units
    int qcnt = 0;   // units with key tiles so far
    bool ok = true;
    int n_next = unit_steps(0);
    for (int r = 0; ok && r < rounds; ++r) {
      const int n = n_next;
      if (n > 0) {
        ok = wait_all(&bar.q_full, qcnt & 1);
        ATTN_TRACE_REC(trole, EV_Q_FULL, qcnt);
#pragma unroll
        for (int si = 0; si < kSubPerWarp && ok; ++si) {
          const int s = s_first + si;
          ok = wait_all(&bar.k_full[slot_of(gstep, s)], phase_of(gstep, s));
          if (!ok) break;
          tc_fence_after();
          if (elect_one_sync()) {
            if constexpr (!kHalfTiles<DECODE, MOD>) {
              qk_mmas(s, slot_of(gstep, s), n == 1);
            } else {
              qk_half_mmas(s, slot_of(gstep, s), 0, false);
              qk_half_mmas(s, slot_of(gstep, s), 1, n == 1);
            }
          }
          __syncwarp();
        }
      }
      n_next = unit_steps(r + 1);
      if (n == 0) continue;
      for (int j = 0; ok && j < n; ++j) {
        const int g = gstep + j;
        const bool more = j + 1 < n;
        constexpr int kHalves = kHalfTiles<DECODE, MOD> ? 2 : 1;
#pragma unroll
        for (int h = 0; h < kHalves && ok; ++h) {
#pragma unroll
          for (int si = 0; si < kSubPerWarp; ++si) {
            const int s = s_first + si;
            const int slot = slot_of(g, s), nslot = slot_of(g + 1, s);
            const uint32_t va = v_lo + (uint32_t)slot * kTileUnits;
            if (h == 0 && !wait_all(&bar.v_full[slot], phase_of(g, s))) { ok = false; break; }
            if (h == 0 && more && !wait_all(&bar.k_full[nslot], phase_of(g + 1, s))) { ok = false; break; }
            ATTN_TRACE_REC(trole, EV_P_WAIT, (g << 1) | s);
            uint64_t* pbar = h == 0 ? &bar.p_ready[s] : &bar.p_b_ready[s];
            if (!wait_spin_all(pbar, g & 1)) { ok = false; break; }
            // The first PV of a unit overwrites O(s): the previous unit's epilogue must have read it.
            if (j == 0 && h == 0 && qcnt > 0 && !wait_all(&bar.o_free[s], (qcnt - 1) & 1)) { ok = false; break; }
            if (!take_turn(s)) { ok = false; break; }
            tc_fence_after();
            ATTN_TRACE_REC(trole, EV_PV, (g << 1) | s);
            if (elect_one_sync()) {
              if constexpr (kHalfTiles<DECODE, MOD>) {
                // PV over keys 64h..64h+63: P from S(s) columns [64h, 64h+32), V rows 64h..
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                  mma_ts(tmem + 256 + s * L::kOCols, tmem + s * 128 + 64 * h + kk * 8,
                         sdesc_join(va + (((4 * h + kk) * 16 * 128) >> 4), kHi), idesc_pv,
                         (j == 0 && h == 0 && kk == 0) ? 0u : 1u);
                if (h == 0) mma_commit(&bar.pv_a_done[s]);
                if (h == 1 && !more) mma_commit(&bar.o_done[s]);
                if (h == 1) mma_commit(&bar.v_empty[slot]);
                if (more) qk_half_mmas(s, nslot, h, h == 1 && j + 2 == n);
              } else {
#pragma unroll
                for (int kk = 0; kk < kKeys / 16; ++kk)
                  mma_ts(tmem + 256 + s * L::kOCols, tmem + s * 128 + kk * 8,
                         sdesc_join(va + ((kk * 16 * 128) >> 4), kHi), idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
                if (!more) mma_commit(&bar.o_done[s]);
                mma_commit(&bar.v_empty[slot]);
                if (more) qk_mmas(s, nslot, j + 2 == n);
              }
            }
            __syncwarp();
            pass_turn(s);
            ++batch;
            ATTN_TRACE_REC(trole, EV_PV_ISSUED, (g << 1) | s);
          }
        }
      }
      gstep += n;
      ++qcnt;
    }
    ATTN_TRACE_REC(trole, EV_MMA_END, gstep);
    // Every MMA of this warp must be complete before TMEM is released.
    if (elect_one_sync()) mma_commit(&bar.final_mma[s_first]);
    __syncwarp();
    mbar_wait_timeout(&bar.final_mma[s_first], 0);
  } else if (warp >= kMmaWarp) {
    regs_decrease<kControlRegs>();  // idle: completes the third warpgroup
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
    // The next round's unit is set up while this warp waits for the current
    // unit's last PV (once-per-unit code, usually refetched into the
    // instruction cache), not after the epilogue.
    int u_next;
    Work w_next;
    TileWalker tw_next;
    int n_next = 0;
    auto setup = [&](int r) {
      u_next = r < rounds ? unit_of(r) : -1;
      if (u_next >= 0) {
        w_next = map_work<DECODE>(a, u_next);
        n_next = walker_init<DECODE, BM, kDescWalk<DECODE, MOD>>(a, w_next, tw_next);
      }
    };
    setup(0);
    for (int r = 0; ok && r < rounds; ++r) {
      const bool have_unit = u_next >= 0;
      const Work w = w_next;
      TileWalker tw = tw_next;
      const int n = have_unit ? n_next : 0;
      RowState st;
      st.m = -__int_as_float(0x7f800000);
      st.l = 0.f;
      if (DECODE) tw.t += s;
      for (int j = 0; j < n; ++j) {
        const int t = tw.t;
        const int cls = tile_class<DECODE, BM>(a, w, s, t);
        ATTN_TRACE_REC(warp, EV_S_WAIT, gstep + j);
        if (!wait_spin_all(&bar.s_ready[s], (gstep + j) & 1)) { ok = false; break; }
        tc_fence_after();
        ATTN_TRACE_REC(warp, EV_S_READY, (gstep + j) | (cls << 20));
        if constexpr (!kHalfTiles<DECODE, MOD>) {
          softmax_step<D, DECODE, MOD, BM>(a, w, s, row, t, cls, tS, tO, j == 0, st, &bar.p_ready[s]);
        } else if (!softmax_step_halves<D, MOD, BM>(a, w, s, row, t, cls, tS, tO, j == 0, st, bar, gstep + j,
                                                      abort_flag)) {
          ok = false;
          break;
        }
        ATTN_TRACE_REC(warp, EV_P_DONE, gstep + j);
        if (DECODE)
          tw.t += 2;
        else
          walker_next<BM, kDescWalk<DECODE, MOD>>(tw);
      }
      if (!ok) break;
      setup(r + 1);
      if (!have_unit) continue;
      ATTN_TRACE_REC(warp, EV_O_WAIT, qcnt);
      if (n > 0) {
        bool got = wait_all(&bar.o_done[s], qcnt & 1);
        if (DECODE && s == 0) got = got && wait_all(&bar.o_done[1], qcnt & 1);
        if (!got) break;
        tc_fence_after();
      }
      ATTN_TRACE_REC(warp, EV_EPI_BEGIN, qcnt);
      // A unit without key tiles still writes its (all-masked) outputs.
      if (!epilogue<D, DECODE>(a, &map_o, w, s, row, lane_base, n > 0, st, extra, bar, qcnt, abort_flag)) break;
      ATTN_TRACE_REC(warp, EV_EPI_END, qcnt);
      if (n == 0) continue;
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
    // Output stores complete before the CTA (and its staging memory) goes away.
    if (lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) {
    __syncwarp();
    tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0 && bar.abort_flag && a.status) atomicOr(a.status, DEV_TIMEOUT);
  if (threadIdx.x == 0) ATTN_TRACE_REC(0, EV_KERNEL_END, 0);
}

}  // namespace attn_kernels
