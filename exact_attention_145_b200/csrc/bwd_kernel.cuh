// bwd_kernel.cuh - attention backward for sm_100a (attn_bwd): dQ, dK, dV of
// O = softmax(scale * Q K^T + mask) V for an upstream gradient dO, with the
// forward's log-sum-exp as input. The FlashAttention overview ("Examples")
// names this backward pass and its deterministic option; the kernels here
// are deterministic by construction: every output element is accumulated in
// a fixed order, with no atomics.
//
// With P = exp(scale * S - LSE) (S = Q K^T, masked entries 0), the chain rule
// gives dV = P^T dO, dP = dO V^T, dS = P o (dP - delta) with delta_i =
// dO_i . O_i, dQ = scale * dS K and dK = scale * dS^T Q. Four kernels:
//   delta_kernel   delta_i for every (b, h, i) on CUDA cores; its last block
//                  writes the dK/dV work plan (below);
//   dkdv kernel    one work unit per piece of a (b, KV head, 128-key tile):
//                  a contiguous range of the tile's steps (query tile x query
//                  head of the group), recomputing S^T = K Q^T and
//                  dP^T = V dO^T in TMEM, writing P^T and dS^T back to TMEM
//                  as bf16 and accumulating dV += P^T dO and dK += dS^T Q
//                  there (tcgen05, A from TMEM);
//   dkdv reduce    sums the fp32 partials of key tiles cut into several
//                  pieces, in piece order;
//   dq kernel      one work unit per (b, query head, 128-row tile): loops over
//                  the key tiles, S = Q K^T and dP = dO V^T in TMEM, dS back
//                  to TMEM as bf16, dQ += dS K.
// Pieces balance the causal triangle: key tile 0 meets every query tile,
// the last key tile one, so whole tiles as units would leave the first
// CTAs with several times the mean work.
// Warp roles (320 threads): warps 0-7 compute (warp w: TMEM lanes
// 32 (w % 4) .. +31 = the tile's rows, columns half w / 4), warp 8 MMA issue
// (owns TMEM), warp 9 TMA producer. Every wait is bounded (sm100.cuh).
// Each step runs as two column halves with their own barriers: the tensor
// pipe computes half B's S / dP while half A's warps compute, then half A's
// accumulation and the next step's half A products while half B computes.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "sm100.cuh"

namespace attn_bwd_kernels {

using namespace attn_sm100;

constexpr int kTile = 128;  // rows of a Q tile, keys of a K/V tile
constexpr int kBwdThreads = 320;
constexpr int kBCompute = 256;  // compute threads: two per tile row
constexpr int kBMmaWarp = 8;
constexpr int kBTmaWarp = 9;
constexpr int kPlanThreads = 256;
constexpr float kLog2eB = 1.4426950408889634f;
enum : int { BMASK_NONE = 0, BMASK_CAUSAL = 1, BMASK_WINDOW = 2 };
enum : int { BDEV_TIMEOUT = 1 };

// Steps of key tile t in the dK/dV pass: (query tiles that meet it) x g.
// *qlo receives the first such query tile. Shared by the host (workspace
// sizing, grid) and the plan block, so both count the same pieces.
__host__ __device__ inline int kv_tile_steps(int Sq, int Skv, int g, int mask, int wl, int wr, int q_offset, int t,
                                             int* qlo) {
  const long long k0 = (long long)t * kTile;
  const long long kend = (long long)(t + 1) * kTile < (long long)Skv ? (long long)(t + 1) * kTile : (long long)Skv;
  const long long k1 = kend - 1;
  long long lo = 0, hi = (long long)Sq - 1;
  if (mask != BMASK_NONE) {
    // key k is seen by q_pos in [k - wr, k + wl]; q_pos = i + q_offset
    if (wr >= 0 && k0 - wr - q_offset > lo) lo = k0 - wr - q_offset;
    if (wl >= 0 && k1 + wl - q_offset < hi) hi = k1 + wl - q_offset;
  }
  if (hi < lo) {
    *qlo = 0;
    return 0;
  }
  *qlo = (int)(lo / kTile);
  return (int)(hi / kTile - lo / kTile + 1) * g;
}

// Pieces of a key tile with n steps under a piece cap: at least one (a tile
// no query sees still writes its zero gradients).
__host__ __device__ inline int kv_tile_pieces(int n, int cap) { return n <= cap ? 1 : (n + cap - 1) / cap; }

struct BwdArgs {
  int B, Hq, Hkv, Sq, Skv, g;
  float scale, scale_log2;
  int mask, wl, wr, q_offset;  // window form: q_pos - wl <= key <= q_pos + wr (-1 = unbounded side)
  int nQ, nK;
  const float* lse;    // [B][Hq][Sq] natural log (from the forward)
  const float* delta;  // [B][Hq][Sq] (workspace, written by delta_kernel)
  __nv_bfloat16 *dq, *dk, *dv;
  int64_t dq_sb, dq_ss, dq_sh, dk_sb, dk_ss, dk_sh, dv_sb, dv_ss, dv_sh;
  // dK/dV plan (workspace, written by the delta kernel's last block):
  const int4* pieces;  // [n_pieces] {key tile, first step, end step, partial slot or -1}
  const int2* tiles;   // [nK] {pieces of the tile, first partial slot or -1}
  float* part;         // [B * Hkv][n_slots][2][D / 4][128] float4: fp32 partial dV, dK (dK without the scale),
                       // row-interleaved so that a warp's rows are one contiguous 512-byte store
  int n_pieces, n_slots, cap;
  int n_units;
  int* status;
};

// ---------------------------------------------------------------- delta + plan
// delta[b][h][i] = sum_d dO[b,i,h,d] * O[b,i,h,d]; D / 8 threads per row,
// 16-byte loads. The last block writes the dK/dV plan instead.
struct DeltaArgs {
  const __nv_bfloat16 *o, *dout;
  int64_t o_sb, o_ss, o_sh, do_sb, do_ss, do_sh;
  int B, Hq, Sq, D;
  float* delta;
  int delta_blocks;
  BwdArgs plan;  // mask and sizes for the plan; pieces / tiles written through const_cast
};

__device__ __forceinline__ float dot8_bf16(uint4 x, uint4 y) {
  const __nv_bfloat162* a = reinterpret_cast<const __nv_bfloat162*>(&x);
  const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&y);
  float acc = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 u = __bfloat1622float2(a[i]), v = __bfloat1622float2(b[i]);
    acc = fmaf(u.x, v.x, acc);
    acc = fmaf(u.y, v.y, acc);
  }
  return acc;
}

// Block-wide exclusive scan of two counters (kPlanThreads threads).
__device__ __forceinline__ void block_scan2(int& a, int& b, int* sh) {
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
  int ia = a, ib = b;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int ya = __shfl_up_sync(0xffffffffu, ia, off), yb = __shfl_up_sync(0xffffffffu, ib, off);
    if (lane >= off) {
      ia += ya;
      ib += yb;
    }
  }
  if (lane == 31) {
    sh[warp] = ia;
    sh[32 + warp] = ib;
  }
  __syncthreads();
  int ba = 0, bb = 0;
  for (int w = 0; w < warp; ++w) {
    ba += sh[w];
    bb += sh[32 + w];
  }
  a = ba + ia - a;
  b = bb + ib - b;
}

__device__ void write_plan(const BwdArgs& p) {
  __shared__ int sh[64];
  const int nK = p.nK;
  const int per = (nK + kPlanThreads - 1) / kPlanThreads;
  const int t0 = min((int)threadIdx.x * per, nK), t1 = min(t0 + per, nK);
  int np_sum = 0, slot_sum = 0, qlo;
  for (int t = t0; t < t1; ++t) {
    const int np = kv_tile_pieces(kv_tile_steps(p.Sq, p.Skv, p.g, p.mask, p.wl, p.wr, p.q_offset, t, &qlo), p.cap);
    np_sum += np;
    slot_sum += np > 1 ? np : 0;
  }
  int ps = np_sum, ss = slot_sum;
  block_scan2(ps, ss, sh);
  int4* pieces = const_cast<int4*>(p.pieces);
  int2* tiles = const_cast<int2*>(p.tiles);
  for (int t = t0; t < t1; ++t) {
    const int n = kv_tile_steps(p.Sq, p.Skv, p.g, p.mask, p.wl, p.wr, p.q_offset, t, &qlo);
    const int np = kv_tile_pieces(n, p.cap);
    tiles[t] = make_int2(np, np > 1 ? ss : -1);
    for (int j = 0; j < np; ++j)
      pieces[ps + j] = make_int4(t, (int)((long long)j * n / np), (int)((long long)(j + 1) * n / np), np > 1 ? ss + j : -1);
    ps += np;
    ss += np > 1 ? np : 0;
  }
}

__global__ void __launch_bounds__(256) delta_kernel(const DeltaArgs a) {
  if ((int)blockIdx.x == a.delta_blocks) {
    write_plan(a.plan);
    return;
  }
  const int tpr = a.D / 8;  // threads per row
  const int rows_per_block = 256 / tpr;
  const int64_t row = (int64_t)blockIdx.x * rows_per_block + threadIdx.x / tpr;
  const int part = threadIdx.x % tpr;
  const bool live = row < (int64_t)a.B * a.Hq * a.Sq;
  float acc = 0.f;
  int i = 0, h = 0, b = 0;
  if (live) {
    i = (int)(row % a.Sq);
    h = (int)((row / a.Sq) % a.Hq);
    b = (int)(row / ((int64_t)a.Sq * a.Hq));
    const __nv_bfloat16* o = a.o + b * a.o_sb + (int64_t)i * a.o_ss + (int64_t)h * a.o_sh + part * 8;
    const __nv_bfloat16* d = a.dout + b * a.do_sb + (int64_t)i * a.do_ss + (int64_t)h * a.do_sh + part * 8;
    acc = dot8_bf16(*reinterpret_cast<const uint4*>(o), *reinterpret_cast<const uint4*>(d));
  }
  for (int off = tpr / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (live && part == 0) a.delta[((int64_t)b * a.Hq + h) * a.Sq + i] = acc;
}

// ---------------------------------------------------------------- masks
// Key tiles [lo, hi] that meet query tile qt.
__device__ __forceinline__ bool k_range_for_q(const BwdArgs& a, int qt, int& lo, int& hi) {
  const long q0 = (long)qt * kTile + a.q_offset, q1 = min((long)(qt + 1) * kTile, (long)a.Sq) - 1 + a.q_offset;
  long klo = 0, khi = (long)a.Skv - 1;
  if (a.mask != BMASK_NONE) {
    if (a.wl >= 0) klo = max(klo, q0 - a.wl);
    if (a.wr >= 0) khi = min(khi, q1 + a.wr);
  }
  if (khi < klo) return false;
  lo = (int)(klo / kTile);
  hi = (int)(khi / kTile);
  return true;
}

// A (query tile qt, key tile t) pair needs per-element masking unless every
// in-tile pair is allowed and neither side is ragged.
__device__ __forceinline__ bool pair_full(const BwdArgs& a, int qt, int t) {
  const long q0 = (long)qt * kTile, q1 = (long)(qt + 1) * kTile - 1;
  const long k0 = (long)t * kTile, k1 = (long)(t + 1) * kTile - 1;
  if (q1 >= a.Sq || k1 >= a.Skv) return false;
  if (a.mask == BMASK_NONE) return true;
  bool full = true;
  if (a.wl >= 0 && k0 < q1 + a.q_offset - a.wl) full = false;
  if (a.wr >= 0 && k1 > q0 + a.q_offset + a.wr) full = false;
  return full;
}

// Bit e of the result: element e of a 32-wide chunk starting at position
// c0 on the other axis is allowed, given that the thread's own position is
// allowed exactly for other-axis positions in [lo, hi].
__device__ __forceinline__ uint32_t range_bits(long lo, long hi, long c0) {
  const long a = lo - c0, b = hi - c0;
  if (b < 0 || a > 31 || b < a) return 0u;
  const int l = (int)max(a, 0l), h = (int)min(b, 31l);
  return (0xffffffffu >> (31 - h)) & (0xffffffffu << l);
}

// ---------------------------------------------------------------- layout
template <int D>
struct BLayout {
  static constexpr int kTileBytes = kTile * D * 2;    // one operand tile (128 rows x D bf16)
  static constexpr int kChunk = kTile * 64 * 2;       // one 128-row x 64-column SW128 box
  // dkdv: K, V of the unit, then a 2-slot ring of (Q, dO) per step.
  // dq: Q, dO of the unit, then a 2-slot ring of (K, V) per step.
  static constexpr int kFixOff = 0;                   // two unit tiles
  static constexpr int kRingOff = 2 * kTileBytes;     // 2 slots x two step tiles
  static constexpr int kVecOff = kRingOff + 4 * kTileBytes;  // dkdv: 2 slots x 2 halves x (log2e*LSE, delta) x 64 floats
  static constexpr int kBarOff = kVecOff + 2 * 2 * kTile * 4;
  // Each CTA allocates all 512 TMEM columns, so two CTAs must never share an
  // SM: the request is padded past half of the SM's 228 KB of shared memory.
  static constexpr int kUsedBytes = kBarOff + 1024 + 1024;
  static constexpr int kSmemBytes = kUsedBytes > 120 * 1024 ? kUsedBytes : 120 * 1024;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
  static_assert(kVecOff % 1024 == 0, "operand tiles stay 1024-byte aligned");
};

struct BBarriers {
  uint64_t fix_full, fix_empty;  // unit tiles loaded / released
  uint64_t ring_full[2], ring_empty[2];
  uint64_t mm1_ready[2];   // per column half: the step's S / dP products are in TMEM
  uint64_t comp_ready[2];  // per half: its warps wrote P^T / dS^T (dkdv) or dS (dq): 128 arrivals
  uint64_t acc_done;       // the unit's accumulators are final
  uint64_t acc_free;       // the epilogue read them: 256 arrivals
  uint64_t vec_ready[2][2];  // dkdv, [slot][half]: the half's LSE / delta columns are in shared memory
  uint64_t final_mma;
  uint32_t tmem_base;
  int abort_flag;
};

// The bf16 result of 32-column chunk c (P^T / dS^T / dS) is packed into the
// first 16 columns of the chunk's own source columns, so that the two
// column halves of a tile never write where the other half still reads.
// A-operand column of the TS MMA over rows 16 kk .. 16 kk + 15 of the
// contraction:
__device__ __forceinline__ uint32_t packed_col(int kk) { return 32u * (uint32_t)(kk >> 1) + 8u * (uint32_t)(kk & 1); }

// ---------------------------------------------------------------- work maps
// dkdv unit u -> piece pid = u / (B * Hkv) of group (b, hk) = u % (B * Hkv).
// Pieces are numbered by key tile, so the causal heavy tiles come first.
struct KvUnit {
  int b, hk, t, qlo, s0, n, slot;  // steps s0 .. s0 + n - 1; slot >= 0: write fp32 partials
};
__device__ __forceinline__ KvUnit kv_unit(const BwdArgs& a, int u) {
  KvUnit w;
  const int per = a.B * a.Hkv;
  const int pid = u / per, grp = u % per;
  w.b = grp / a.Hkv;
  w.hk = grp % a.Hkv;
  const int4 pc = a.pieces[pid];
  w.t = pc.x;
  w.s0 = pc.y;
  w.n = pc.z - pc.y;
  w.slot = pc.w;
  kv_tile_steps(a.Sq, a.Skv, a.g, a.mask, a.wl, a.wr, a.q_offset, w.t, &w.qlo);
  return w;
}
// dq unit u -> (b, h, q tile qt); last q tiles first (the most key tiles).
struct QUnit {
  int b, h, qt, klo, n;
};
__device__ __forceinline__ QUnit q_unit(const BwdArgs& a, int u) {
  QUnit w;
  const int per = a.B * a.Hq;
  w.qt = a.nQ - 1 - u / per;
  const int r = u % per;
  w.b = r / a.Hq;
  w.h = r % a.Hq;
  int lo = 0, hi = -1;
  w.n = k_range_for_q(a, w.qt, lo, hi) ? hi - lo + 1 : 0;
  w.klo = lo;
  return w;
}

__device__ __forceinline__ float bex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---------------------------------------------------------------- dK / dV
// TMEM columns: S^T [0, 128), dP^T [128, 256), dV [256, 256 + D), dK [256 + D, 256 + 2D).
// MMA order per step, by 64-query halves A / B: S^T_A dP^T_A S^T_B dP^T_B |
// (compute A) | dV_A dK_A S^T_A(next) dP^T_A(next) | (compute B) | dV_B dK_B ...
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                         const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_do,
                         const BwdArgs a) {
  using L = BLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  BBarriers& bar = *reinterpret_cast<BBarriers*>(smem + L::kBarOff);
  const int warp = threadIdx.x / 32;
  volatile int* abort_flag = &bar.abort_flag;
  if (threadIdx.x == 0) {
    bar.abort_flag = 0;
    mbar_init(&bar.fix_full, 1);
    mbar_init(&bar.fix_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar.ring_full[i], 1);
      mbar_init(&bar.ring_empty[i], 1);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(&bar.mm1_ready[h], 1);
      mbar_init(&bar.comp_ready[h], kTile);
      mbar_init(&bar.vec_ready[0][h], kTile);
      mbar_init(&bar.vec_ready[1][h], kTile);
    }
    mbar_init(&bar.acc_done, 1);
    mbar_init(&bar.acc_free, kBCompute);
    mbar_init(&bar.final_mma, 1);
    fence_barrier_init();
  }
  if (warp == kBMmaWarp) {
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
  auto wait_all = [&](uint64_t* b, uint32_t par) { return __all_sync(0xffffffffu, mbar_wait(b, par, abort_flag)); };
  auto wait_spin_all = [&](uint64_t* b, uint32_t par) {
    return __all_sync(0xffffffffu, mbar_wait_spin(b, par, abort_flag));
  };
  // step s of a unit: q tile qlo + s / g, query head hk * g + s % g
  if (warp == kBTmaWarp) {
    // ------------------------------------------------------------ producer
    if (elect_one_sync()) {
      tma_prefetch_desc(&map_q);
      tma_prefetch_desc(&map_do);
    }
    __syncwarp();
    int ucnt = 0, gstep = 0;
    bool ok = true;
    for (int r = 0; ok && r < rounds; ++r) {
      const int u = unit_of(r);
      if (u < 0) continue;
      const KvUnit w = kv_unit(a, u);
      if (w.n == 0) continue;
      if (ucnt > 0 && !wait_all(&bar.fix_empty, (ucnt - 1) & 1)) { ok = false; break; }
      if (elect_one_sync()) {
        mbar_arrive_expect_tx(&bar.fix_full, 2 * L::kTileBytes);
        for (int c = 0; c < D / 64; ++c) {
          tma_load_4d(smem + L::kFixOff + c * L::kChunk, &map_k, &bar.fix_full, c * 64, w.t * kTile, w.hk, w.b);
          tma_load_4d(smem + L::kFixOff + L::kTileBytes + c * L::kChunk, &map_v, &bar.fix_full, c * 64, w.t * kTile,
                      w.hk, w.b);
        }
      }
      __syncwarp();
      ++ucnt;
      for (int s = w.s0; s < w.s0 + w.n; ++s, ++gstep) {
        const int slot = gstep & 1, use = gstep >> 1;
        if (use > 0 && !wait_all(&bar.ring_empty[slot], (use - 1) & 1)) { ok = false; break; }
        const int qt = w.qlo + s / a.g, h = w.hk * a.g + s % a.g;
        if (elect_one_sync()) {
          uint64_t* fb = &bar.ring_full[slot];
          mbar_arrive_expect_tx(fb, 2 * L::kTileBytes);
          uint8_t* base = smem + L::kRingOff + slot * 2 * L::kTileBytes;
          for (int c = 0; c < D / 64; ++c) {
            tma_load_4d(base + c * L::kChunk, &map_q, fb, c * 64, qt * kTile, h, w.b);
            tma_load_4d(base + L::kTileBytes + c * L::kChunk, &map_do, fb, c * 64, qt * kTile, h, w.b);
          }
        }
        __syncwarp();
      }
    }
    if (*abort_flag) {
      if (ucnt > 0) mbar_wait_timeout(&bar.fix_full, (ucnt - 1) & 1);
      for (int k = max(0, gstep - 2); k < gstep; ++k) mbar_wait_timeout(&bar.ring_full[k & 1], (k >> 1) & 1);
    }
  } else if (warp == kBMmaWarp) {
    // ------------------------------------------------------------ MMA issue
    constexpr uint32_t kHi = sdesc_sw128_hi(1024);
    constexpr uint32_t idesc_mm1 = idesc_bf16_f32(128, 64, 0, 0);  // K-major A and B, one 64-query half
    constexpr uint32_t idesc_acc = idesc_bf16_f32(128, D, 0, 1);   // B MN-major (rows x D tiles)
    constexpr uint32_t kTileUnits = L::kTileBytes >> 4;
    constexpr uint32_t kHalfRows = (64 * 128) >> 4;                  // 64 rows of a SW128 chunk
    const uint32_t k_lo = sdesc_sw128_lo(smem_u32(smem + L::kFixOff), 16);
    const uint32_t v_lo = k_lo + kTileUnits;
    const uint32_t ring_lo = sdesc_sw128_lo(smem_u32(smem + L::kRingOff), 16);
    const uint32_t ring_mn = sdesc_sw128_lo(smem_u32(smem + L::kRingOff), L::kChunk);
    // Half h of the step in ring slot `slot`: S^T = K Q^T for queries 64h..64h+63
    // into columns [64h, 64h + 64), dP^T = V dO^T into [128 + 64h, ...).
    auto mm1_half = [&](int slot, int h) {
      const uint32_t qa = ring_lo + (uint32_t)slot * 2 * kTileUnits + (uint32_t)h * kHalfRows, da = qa + kTileUnits;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = ((kk / 4) * L::kChunk + (kk % 4) * 32) >> 4;
        mma_ss(tmem + 64 * h, sdesc_join(k_lo + off, kHi), sdesc_join(qa + off, kHi), idesc_mm1, kk > 0);
      }
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = ((kk / 4) * L::kChunk + (kk % 4) * 32) >> 4;
        mma_ss(tmem + 128 + 64 * h, sdesc_join(v_lo + off, kHi), sdesc_join(da + off, kHi), idesc_mm1, kk > 0);
      }
      mma_commit(&bar.mm1_ready[h]);
    };
    // Half h's accumulation: dV += P^T dO and dK += dS^T Q over queries 64h..64h+63.
    auto acc_half = [&](int slot, int h, bool first) {
      const uint32_t qmn = ring_mn + (uint32_t)slot * 2 * kTileUnits, dmn = qmn + kTileUnits;
#pragma unroll
      for (int k4 = 0; k4 < 4; ++k4) {
        const int kk = 4 * h + k4;
        mma_ts(tmem + 256, tmem + packed_col(kk), sdesc_join(dmn + ((kk * 16 * 128) >> 4), kHi), idesc_acc,
               (!first || kk > 0) ? 1u : 0u);
      }
#pragma unroll
      for (int k4 = 0; k4 < 4; ++k4) {
        const int kk = 4 * h + k4;
        mma_ts(tmem + 256 + D, tmem + 128 + packed_col(kk), sdesc_join(qmn + ((kk * 16 * 128) >> 4), kHi),
               idesc_acc, (!first || kk > 0) ? 1u : 0u);
      }
    };
    int ucnt = 0, gstep = 0;
    bool ok = true;
    for (int r = 0; ok && r < rounds; ++r) {
      const int u = unit_of(r);
      if (u < 0) continue;
      const KvUnit w = kv_unit(a, u);
      if (w.n == 0) continue;
      ok = wait_all(&bar.fix_full, ucnt & 1) && wait_all(&bar.ring_full[gstep & 1], (gstep >> 1) & 1);
      if (!ok) break;
      tc_fence_after();
      if (elect_one_sync()) {
        mm1_half(gstep & 1, 0);
        mm1_half(gstep & 1, 1);
      }
      __syncwarp();
      for (int s = 0; s < w.n; ++s) {
        const int g = gstep + s, slot = g & 1;
        const bool more = s + 1 < w.n;
        // half A: its accumulation, then the next step's half A products
        if (!wait_spin_all(&bar.comp_ready[0], g & 1)) { ok = false; break; }
        // The unit's first accumulation overwrites dV / dK: the previous
        // unit's epilogue must have read them.
        if (s == 0 && ucnt > 0 && !wait_all(&bar.acc_free, (ucnt - 1) & 1)) { ok = false; break; }
        if (more && !wait_all(&bar.ring_full[(g + 1) & 1], ((g + 1) >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        if (elect_one_sync()) {
          acc_half(slot, 0, s == 0);
          if (more) mm1_half((g + 1) & 1, 0);
        }
        __syncwarp();
        // half B: its accumulation, the slot's release, the next half B products
        if (!wait_spin_all(&bar.comp_ready[1], g & 1)) { ok = false; break; }
        tc_fence_after();
        if (elect_one_sync()) {
          acc_half(slot, 1, s == 0);
          mma_commit(&bar.ring_empty[slot]);
          if (more) {
            mm1_half((g + 1) & 1, 1);
          } else {
            mma_commit(&bar.acc_done);
            mma_commit(&bar.fix_empty);
          }
        }
        __syncwarp();
      }
      gstep += w.n;
      ++ucnt;
    }
    if (elect_one_sync()) mma_commit(&bar.final_mma);
    __syncwarp();
    mbar_wait_timeout(&bar.final_mma, 0);
  } else {
    // ------------------------------------------------------------ compute
    const int row = threadIdx.x % kTile;  // key row of the tile = TMEM lane
    const int half = warp / 4;            // columns [64 half, 64 half + 64) of S^T / dP^T
    const uint32_t lane_base = tmem + ((uint32_t)((warp % 4) * 32) << 16);
    int ucnt = 0, gstep = 0;
    bool ok = true;
    const float NEG_INF = -__int_as_float(0x7f800000);
    for (int r = 0; ok && r < rounds; ++r) {
      const int u = unit_of(r);
      if (u < 0) continue;
      const KvUnit w = kv_unit(a, u);
      const long key = (long)w.t * kTile + row;
      const bool real = key < a.Skv;
      const int c_lo = half * (D / 2);  // this thread's output columns [c_lo, c_lo + D / 2)
      if (w.n == 0) {
        // no query sees these keys: their gradients are exactly zero
        if (real) {
          __nv_bfloat16* dvr = a.dv + w.b * a.dv_sb + key * a.dv_ss + (int64_t)w.hk * a.dv_sh + c_lo;
          __nv_bfloat16* dkr = a.dk + w.b * a.dk_sb + key * a.dk_ss + (int64_t)w.hk * a.dk_sh + c_lo;
          for (int c = 0; c < D / 2; c += 8) {
            *reinterpret_cast<uint4*>(dvr + c) = make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4*>(dkr + c) = make_uint4(0, 0, 0, 0);
          }
        }
        continue;
      }
      // queries that see this key: q_pos in [key - wr, key + wl], q_pos = i + q_offset
      long qlo_i = 0, qhi_i = (long)a.Sq - 1;
      if (a.mask != BMASK_NONE) {
        if (a.wr >= 0) qlo_i = max(qlo_i, key - a.wr - a.q_offset);
        if (a.wl >= 0) qhi_i = min(qhi_i, key + a.wl - a.q_offset);
      }
      if (!real) qhi_i = -1;
      // Column values of a step for this half's 64 queries (log2e * LSE and
      // delta): thread row fetches LSE (rows 0-63) or delta (rows 64-127) of
      // query qt*128 + 64 half + row % 64. The global load for step s + 1 is
      // issued during step s, so its latency is off the per-step chain.
      auto column_value = [&](int s) -> float {
        const int qt = w.qlo + (w.s0 + s) / a.g, h = w.hk * a.g + (w.s0 + s) % a.g;
        const int typ = row / 64, qi = qt * kTile + 64 * half + row % 64;
        // stored negated: -log2e * LSE (-inf for a row with no allowed key
        // or past Sq, so its weights come out +0) and -delta
        float val = typ == 0 ? NEG_INF : 0.f;
        if (qi < a.Sq) {
          const int64_t ix = ((int64_t)w.b * a.Hq + h) * a.Sq + qi;
          if (typ == 0) {
            const float l = __ldg(a.lse + ix);
            val = l == NEG_INF ? NEG_INF : -l * kLog2eB;
          } else {
            val = -__ldg(a.delta + ix);
          }
        }
        return val;
      };
      float next_val = column_value(0);
      for (int s = 0; s < w.n; ++s) {
        const int g = gstep + s, slot = g & 1;
        const int qt = w.qlo + (w.s0 + s) / a.g;
        // the half's own double-buffered array, published by a bounded
        // mbarrier (128 arrivals)
        float* vec = reinterpret_cast<float*>(smem + L::kVecOff) + (slot * 2 + half) * kTile;
        vec[row] = next_val;
        mbar_arrive(&bar.vec_ready[slot][half]);
        if (s + 1 < w.n) next_val = column_value(s + 1);
        if (!wait_spin_all(&bar.mm1_ready[half], g & 1)) { ok = false; break; }
        if (!wait_spin_all(&bar.vec_ready[slot][half], (g >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        const bool full = pair_full(a, qt, w.t);
#pragma unroll 1
        for (int cc = 0; cc < 2; ++cc) {
          const int c = 2 * half + cc;
          float x[32], dp[32];
          tmem_ld32f(lane_base + 32 * c, x);
          tmem_ld32f(lane_base + 128 + 32 * c, dp);
          tmem_ld_wait();
          reg_fence_f<32>(x);
          reg_fence_f<32>(dp);
          const uint32_t bits = full ? 0xffffffffu : range_bits(qlo_i, qhi_i, (long)qt * kTile + 32 * c);
          const float4* nl2v = reinterpret_cast<const float4*>(vec + 32 * cc);
          const float4* ndlv = reinterpret_cast<const float4*>(vec + 64 + 32 * cc);
          const float2 SL2 = make_float2(a.scale_log2, a.scale_log2);
          uint32_t pk[16], dk[16];
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) {
            const float4 l4 = nl2v[e4], d4 = ndlv[e4];
            const int e = 4 * e4;
            // P^T = 2^(scale log2e S^T - log2e LSE), dS^T = P^T (dP^T - delta), two columns per op
            const float2 z0 = fma2(make_float2(x[e], x[e + 1]), SL2, make_float2(l4.x, l4.y));
            const float2 z1 = fma2(make_float2(x[e + 2], x[e + 3]), SL2, make_float2(l4.z, l4.w));
            float2 p0 = make_float2(bex2(z0.x), bex2(z0.y)), p1 = make_float2(bex2(z1.x), bex2(z1.y));
            if (!full) {
              p0.x = ((bits >> e) & 1u) ? p0.x : 0.f;
              p0.y = ((bits >> (e + 1)) & 1u) ? p0.y : 0.f;
              p1.x = ((bits >> (e + 2)) & 1u) ? p1.x : 0.f;
              p1.y = ((bits >> (e + 3)) & 1u) ? p1.y : 0.f;
            }
            const float2 ds0 = mul2(p0, add2(make_float2(dp[e], dp[e + 1]), make_float2(d4.x, d4.y)));
            const float2 ds1 = mul2(p1, add2(make_float2(dp[e + 2], dp[e + 3]), make_float2(d4.z, d4.w)));
            pk[2 * e4] = pack_bf16x2(p0.x, p0.y);
            pk[2 * e4 + 1] = pack_bf16x2(p1.x, p1.y);
            dk[2 * e4] = pack_bf16x2(ds0.x, ds0.y);
            dk[2 * e4 + 1] = pack_bf16x2(ds1.x, ds1.y);
          }
          // P^T and dS^T of chunk c -> the first 16 of its own 32 source columns
          tmem_st16(lane_base + 32 * c, *reinterpret_cast<uint32_t(*)[16]>(pk));
          tmem_st16(lane_base + 128 + 32 * c, *reinterpret_cast<uint32_t(*)[16]>(dk));
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bar.comp_ready[half]);
      }
      if (!ok) break;
      // epilogue: dV, dK rows, this thread's half of the columns
      if (!wait_all(&bar.acc_done, ucnt & 1)) break;
      tc_fence_after();
      {
        // tcgen05.ld is warp-collective: every lane loads, only rows of real
        // keys are stored (a ragged tile splits a warp).
        const long krow = real ? key : 0;
        __nv_bfloat16* dvr = a.dv + w.b * a.dv_sb + krow * a.dv_ss + (int64_t)w.hk * a.dv_sh + c_lo;
        __nv_bfloat16* dkr = a.dk + w.b * a.dk_sb + krow * a.dk_ss + (int64_t)w.hk * a.dk_sh + c_lo;
        float* pv = nullptr;
        float* pkp = nullptr;
        if (w.slot >= 0) {
          const int grp = w.b * a.Hkv + w.hk;
          float* base = a.part + ((size_t)grp * a.n_slots + w.slot) * 2 * kTile * D;
          pv = base + ((size_t)(c_lo / 4) * kTile + row) * 4;
          pkp = pv + (size_t)kTile * D;
        }
#pragma unroll 1
        for (int c = 0; c < D / 2; c += 32) {
          float v0[32], k0[32];
          tmem_ld32f(lane_base + 256 + c_lo + c, v0);
          tmem_ld32f(lane_base + 256 + D + c_lo + c, k0);
          tmem_ld_wait();
          reg_fence_f<32>(v0);
          reg_fence_f<32>(k0);
          if (w.slot >= 0) {
            // partial of a split key tile: fp32, every row (the reduction skips ragged rows)
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
              const size_t o4 = (size_t)((c + e) / 4) * kTile * 4;  // next column quad: 128 rows further
              *reinterpret_cast<float4*>(pv + o4) = make_float4(v0[e], v0[e + 1], v0[e + 2], v0[e + 3]);
              *reinterpret_cast<float4*>(pkp + o4) = make_float4(k0[e], k0[e + 1], k0[e + 2], k0[e + 3]);
            }
          } else {
#pragma unroll
            for (int e = 0; real && e < 32; e += 8) {
              uint4 pvv, pkk;
              pvv.x = pack_bf16x2(v0[e], v0[e + 1]);
              pvv.y = pack_bf16x2(v0[e + 2], v0[e + 3]);
              pvv.z = pack_bf16x2(v0[e + 4], v0[e + 5]);
              pvv.w = pack_bf16x2(v0[e + 6], v0[e + 7]);
              pkk.x = pack_bf16x2(k0[e] * a.scale, k0[e + 1] * a.scale);
              pkk.y = pack_bf16x2(k0[e + 2] * a.scale, k0[e + 3] * a.scale);
              pkk.z = pack_bf16x2(k0[e + 4] * a.scale, k0[e + 5] * a.scale);
              pkk.w = pack_bf16x2(k0[e + 6] * a.scale, k0[e + 7] * a.scale);
              *reinterpret_cast<uint4*>(dvr + c + e) = pvv;
              *reinterpret_cast<uint4*>(dkr + c + e) = pkk;
            }
          }
          __syncwarp();  // reconverge before the next warp-collective load
        }
      }
      tc_fence_before();
      mbar_arrive(&bar.acc_free);
      gstep += w.n;
      ++ucnt;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kBMmaWarp) {
    __syncwarp();
    tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0 && bar.abort_flag && a.status) atomicOr(a.status, BDEV_TIMEOUT);
}

// Sums the partials of key tiles that were cut into several pieces, in piece
// order, and writes dV and scale * dK as bf16. Grid (nK, B * Hkv, D / 16),
// 256 threads: thread = (8-column group, row), reading two row-interleaved
// float4 (coalesced over rows) per tile and writing 16 bytes of bf16.
constexpr int kReduceThreads = 256;
template <int D>
__global__ void __launch_bounds__(kReduceThreads) attn_bwd_dkdv_reduce_kernel(const BwdArgs a) {
  const int t = blockIdx.x, grp = blockIdx.y;
  const int2 tl = a.tiles[t];
  if (tl.x <= 1) return;
  const int b = grp / a.Hkv, hk = grp % a.Hkv;
  const size_t tile_elems = (size_t)kTile * D;
  const float* base = a.part + ((size_t)grp * a.n_slots + tl.y) * 2 * tile_elems;
  const int id = blockIdx.z * kReduceThreads + threadIdx.x;  // < 128 * D / 8
  const int row = id % kTile, c8 = id / kTile;
  const size_t o0 = ((size_t)(2 * c8) * kTile + row) * 4, o1 = o0 + (size_t)kTile * 4;
  float sv[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f}, sk[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int j = 0; j < tl.x; ++j) {
    const float* pvj = base + (size_t)j * 2 * tile_elems;
    const float* pkj = pvj + tile_elems;
    const float4 v0 = *reinterpret_cast<const float4*>(pvj + o0), v1 = *reinterpret_cast<const float4*>(pvj + o1);
    const float4 k0 = *reinterpret_cast<const float4*>(pkj + o0), k1 = *reinterpret_cast<const float4*>(pkj + o1);
    sv[0] += v0.x; sv[1] += v0.y; sv[2] += v0.z; sv[3] += v0.w;
    sv[4] += v1.x; sv[5] += v1.y; sv[6] += v1.z; sv[7] += v1.w;
    sk[0] += k0.x; sk[1] += k0.y; sk[2] += k0.z; sk[3] += k0.w;
    sk[4] += k1.x; sk[5] += k1.y; sk[6] += k1.z; sk[7] += k1.w;
  }
  const long key = (long)t * kTile + row;
  if (key >= a.Skv) return;
  const int col = 8 * c8;
  __nv_bfloat16* dvr = a.dv + b * a.dv_sb + key * a.dv_ss + (int64_t)hk * a.dv_sh + col;
  __nv_bfloat16* dkr = a.dk + b * a.dk_sb + key * a.dk_ss + (int64_t)hk * a.dk_sh + col;
  uint4 ov, ok;
  ov.x = pack_bf16x2(sv[0], sv[1]);
  ov.y = pack_bf16x2(sv[2], sv[3]);
  ov.z = pack_bf16x2(sv[4], sv[5]);
  ov.w = pack_bf16x2(sv[6], sv[7]);
  ok.x = pack_bf16x2(sk[0] * a.scale, sk[1] * a.scale);
  ok.y = pack_bf16x2(sk[2] * a.scale, sk[3] * a.scale);
  ok.z = pack_bf16x2(sk[4] * a.scale, sk[5] * a.scale);
  ok.w = pack_bf16x2(sk[6] * a.scale, sk[7] * a.scale);
  *reinterpret_cast<uint4*>(dvr) = ov;
  *reinterpret_cast<uint4*>(dkr) = ok;
}

// ---------------------------------------------------------------- dQ
// TMEM columns: S [0, 128), dP [128, 256), dQ [256, 256 + D). dS (bf16
// pairs) is packed into S's columns. MMA order per step:
// by 64-key halves: S_A dP_A S_B dP_B | (compute A) | dQ_A S_A(next) dP_A(next) | (compute B) | dQ_B ...
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                       const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_do,
                       const BwdArgs a) {
  using L = BLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  BBarriers& bar = *reinterpret_cast<BBarriers*>(smem + L::kBarOff);
  const int warp = threadIdx.x / 32;
  volatile int* abort_flag = &bar.abort_flag;
  if (threadIdx.x == 0) {
    bar.abort_flag = 0;
    mbar_init(&bar.fix_full, 1);
    mbar_init(&bar.fix_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar.ring_full[i], 1);
      mbar_init(&bar.ring_empty[i], 1);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(&bar.mm1_ready[h], 1);
      mbar_init(&bar.comp_ready[h], kTile);
    }
    mbar_init(&bar.acc_done, 1);
    mbar_init(&bar.acc_free, kBCompute);
    mbar_init(&bar.final_mma, 1);
    fence_barrier_init();
  }
  if (warp == kBMmaWarp) {
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
  auto wait_all = [&](uint64_t* b, uint32_t par) { return __all_sync(0xffffffffu, mbar_wait(b, par, abort_flag)); };
  auto wait_spin_all = [&](uint64_t* b, uint32_t par) {
    return __all_sync(0xffffffffu, mbar_wait_spin(b, par, abort_flag));
  };
  if (warp == kBTmaWarp) {
    // ------------------------------------------------------------ producer
    if (elect_one_sync()) {
      tma_prefetch_desc(&map_k);
      tma_prefetch_desc(&map_v);
    }
    __syncwarp();
    int ucnt = 0, gstep = 0;
    bool ok = true;
    for (int r = 0; ok && r < rounds; ++r) {
      const int u = unit_of(r);
      if (u < 0) continue;
      const QUnit w = q_unit(a, u);
      if (w.n == 0) continue;
      const int hk = w.h / a.g;
      if (ucnt > 0 && !wait_all(&bar.fix_empty, (ucnt - 1) & 1)) { ok = false; break; }
      if (elect_one_sync()) {
        mbar_arrive_expect_tx(&bar.fix_full, 2 * L::kTileBytes);
        for (int c = 0; c < D / 64; ++c) {
          tma_load_4d(smem + L::kFixOff + c * L::kChunk, &map_q, &bar.fix_full, c * 64, w.qt * kTile, w.h, w.b);
          tma_load_4d(smem + L::kFixOff + L::kTileBytes + c * L::kChunk, &map_do, &bar.fix_full, c * 64,
                      w.qt * kTile, w.h, w.b);
        }
      }
      __syncwarp();
      ++ucnt;
      for (int s = 0; s < w.n; ++s, ++gstep) {
        const int slot = gstep & 1, use = gstep >> 1;
        if (use > 0 && !wait_all(&bar.ring_empty[slot], (use - 1) & 1)) { ok = false; break; }
        const int t = w.klo + s;
        if (elect_one_sync()) {
          uint64_t* fb = &bar.ring_full[slot];
          mbar_arrive_expect_tx(fb, 2 * L::kTileBytes);
          uint8_t* base = smem + L::kRingOff + slot * 2 * L::kTileBytes;
          for (int c = 0; c < D / 64; ++c) {
            tma_load_4d(base + c * L::kChunk, &map_k, fb, c * 64, t * kTile, hk, w.b);
            tma_load_4d(base + L::kTileBytes + c * L::kChunk, &map_v, fb, c * 64, t * kTile, hk, w.b);
          }
        }
        __syncwarp();
      }
    }
    if (*abort_flag) {
      if (ucnt > 0) mbar_wait_timeout(&bar.fix_full, (ucnt - 1) & 1);
      for (int k = max(0, gstep - 2); k < gstep; ++k) mbar_wait_timeout(&bar.ring_full[k & 1], (k >> 1) & 1);
    }
  } else if (warp == kBMmaWarp) {
    // ------------------------------------------------------------ MMA issue
    constexpr uint32_t kHi = sdesc_sw128_hi(1024);
    constexpr uint32_t idesc_mm1 = idesc_bf16_f32(128, 64, 0, 0);  // one 64-key half
    constexpr uint32_t idesc_acc = idesc_bf16_f32(128, D, 0, 1);
    constexpr uint32_t kTileUnits = L::kTileBytes >> 4;
    constexpr uint32_t kHalfRows = (64 * 128) >> 4;
    const uint32_t q_lo = sdesc_sw128_lo(smem_u32(smem + L::kFixOff), 16);
    const uint32_t do_lo = q_lo + kTileUnits;
    const uint32_t ring_lo = sdesc_sw128_lo(smem_u32(smem + L::kRingOff), 16);
    const uint32_t ring_mn = sdesc_sw128_lo(smem_u32(smem + L::kRingOff), L::kChunk);
    // Half h: S = Q K^T for keys 64h..64h+63 into [64h, 64h + 64), dP = dO V^T into [128 + 64h, ...).
    auto mm1_half = [&](int slot, int h) {
      const uint32_t ka = ring_lo + (uint32_t)slot * 2 * kTileUnits + (uint32_t)h * kHalfRows, va = ka + kTileUnits;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = ((kk / 4) * L::kChunk + (kk % 4) * 32) >> 4;
        mma_ss(tmem + 64 * h, sdesc_join(q_lo + off, kHi), sdesc_join(ka + off, kHi), idesc_mm1, kk > 0);
      }
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = ((kk / 4) * L::kChunk + (kk % 4) * 32) >> 4;
        mma_ss(tmem + 128 + 64 * h, sdesc_join(do_lo + off, kHi), sdesc_join(va + off, kHi), idesc_mm1, kk > 0);
      }
      mma_commit(&bar.mm1_ready[h]);
    };
    // Half h's accumulation: dQ += dS K over keys 64h..64h+63.
    auto acc_half = [&](int slot, int h, bool first) {
      const uint32_t kmn = ring_mn + (uint32_t)slot * 2 * kTileUnits;
#pragma unroll
      for (int k4 = 0; k4 < 4; ++k4) {
        const int kk = 4 * h + k4;
        mma_ts(tmem + 256, tmem + packed_col(kk), sdesc_join(kmn + ((kk * 16 * 128) >> 4), kHi), idesc_acc,
               (!first || kk > 0) ? 1u : 0u);
      }
    };
    int ucnt = 0, gstep = 0;
    bool ok = true;
    for (int r = 0; ok && r < rounds; ++r) {
      const int u = unit_of(r);
      if (u < 0) continue;
      const QUnit w = q_unit(a, u);
      if (w.n == 0) continue;
      ok = wait_all(&bar.fix_full, ucnt & 1) && wait_all(&bar.ring_full[gstep & 1], (gstep >> 1) & 1);
      if (!ok) break;
      tc_fence_after();
      if (elect_one_sync()) {
        mm1_half(gstep & 1, 0);
        mm1_half(gstep & 1, 1);
      }
      __syncwarp();
      for (int s = 0; s < w.n; ++s) {
        const int g = gstep + s, slot = g & 1;
        const bool more = s + 1 < w.n;
        if (!wait_spin_all(&bar.comp_ready[0], g & 1)) { ok = false; break; }
        if (s == 0 && ucnt > 0 && !wait_all(&bar.acc_free, (ucnt - 1) & 1)) { ok = false; break; }
        if (more && !wait_all(&bar.ring_full[(g + 1) & 1], ((g + 1) >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        if (elect_one_sync()) {
          acc_half(slot, 0, s == 0);
          if (more) mm1_half((g + 1) & 1, 0);
        }
        __syncwarp();
        if (!wait_spin_all(&bar.comp_ready[1], g & 1)) { ok = false; break; }
        tc_fence_after();
        if (elect_one_sync()) {
          acc_half(slot, 1, s == 0);
          mma_commit(&bar.ring_empty[slot]);
          if (more) {
            mm1_half((g + 1) & 1, 1);
          } else {
            mma_commit(&bar.acc_done);
            mma_commit(&bar.fix_empty);
          }
        }
        __syncwarp();
      }
      gstep += w.n;
      ++ucnt;
    }
    if (elect_one_sync()) mma_commit(&bar.final_mma);
    __syncwarp();
    mbar_wait_timeout(&bar.final_mma, 0);
  } else {
    // ------------------------------------------------------------ compute
    const int row = threadIdx.x % kTile;  // query row of the tile = TMEM lane
    const int half = warp / 4;            // key columns [64 half, 64 half + 64)
    const uint32_t lane_base = tmem + ((uint32_t)((warp % 4) * 32) << 16);
    const float NEG_INF = -__int_as_float(0x7f800000);
    int ucnt = 0, gstep = 0;
    bool ok = true;
    for (int r = 0; ok && r < rounds; ++r) {
      const int u = unit_of(r);
      if (u < 0) continue;
      const QUnit w = q_unit(a, u);
      const int qi = w.qt * kTile + row;
      const bool valid = qi < a.Sq;
      const int c_lo = half * (D / 2);
      if (w.n == 0) {
        // these queries see no key: their gradient is exactly zero
        if (valid) {
          __nv_bfloat16* dqr = a.dq + w.b * a.dq_sb + (int64_t)qi * a.dq_ss + (int64_t)w.h * a.dq_sh + c_lo;
          for (int c = 0; c < D / 2; c += 8) *reinterpret_cast<uint4*>(dqr + c) = make_uint4(0, 0, 0, 0);
        }
        continue;
      }
      const int64_t rix = ((int64_t)w.b * a.Hq + w.h) * a.Sq + min(qi, a.Sq - 1);
      const float lse = a.lse[rix];
      // negated row values: -log2e * LSE (-inf: no allowed key / past Sq, weights +0) and -delta
      const float nl2 = (!valid || lse == NEG_INF) ? NEG_INF : -lse * kLog2eB;
      const float ndl = -a.delta[rix];
      // keys this query sees: [q_pos - wl, q_pos + wr]
      const long q_pos = (long)qi + a.q_offset;
      long klo_i = 0, khi_i = (long)a.Skv - 1;
      if (a.mask != BMASK_NONE) {
        if (a.wl >= 0) klo_i = max(klo_i, q_pos - a.wl);
        if (a.wr >= 0) khi_i = min(khi_i, q_pos + a.wr);
      }
      if (!valid) khi_i = -1;
      for (int s = 0; s < w.n; ++s) {
        const int g = gstep + s;
        const int t = w.klo + s;
        if (!wait_spin_all(&bar.mm1_ready[half], g & 1)) { ok = false; break; }
        tc_fence_after();
        const bool full = pair_full(a, w.qt, t);
        // both chunks' S and dP columns in one TMEM round trip
        float xs[2][32], dps[2][32];
        tmem_ld32f(lane_base + 64 * half, xs[0]);
        tmem_ld32f(lane_base + 64 * half + 32, xs[1]);
        tmem_ld32f(lane_base + 128 + 64 * half, dps[0]);
        tmem_ld32f(lane_base + 128 + 64 * half + 32, dps[1]);
        tmem_ld_wait();
        reg_fence_f<32>(xs[0]);
        reg_fence_f<32>(xs[1]);
        reg_fence_f<32>(dps[0]);
        reg_fence_f<32>(dps[1]);
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int c = 2 * half + cc;
          const float* x = xs[cc];
          const float* dp = dps[cc];
          const uint32_t bits = full ? 0xffffffffu : range_bits(klo_i, khi_i, (long)t * kTile + 32 * c);
          const float2 SL2 = make_float2(a.scale_log2, a.scale_log2), NL2 = make_float2(nl2, nl2);
          const float2 NDL = make_float2(ndl, ndl);
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            // dS = 2^(scale log2e S - log2e LSE) (dP - delta), two columns per op
            const float2 z = fma2(make_float2(x[e], x[e + 1]), SL2, NL2);
            float2 p = make_float2(bex2(z.x), bex2(z.y));
            if (!full) {
              p.x = ((bits >> e) & 1u) ? p.x : 0.f;
              p.y = ((bits >> (e + 1)) & 1u) ? p.y : 0.f;
            }
            const float2 ds = mul2(p, add2(make_float2(dp[e], dp[e + 1]), NDL));
            pk[e / 2] = pack_bf16x2(ds.x, ds.y);
          }
          // dS of chunk c -> the first 16 of its own 32 source columns
          tmem_st16(lane_base + 32 * c, *reinterpret_cast<uint32_t(*)[16]>(pk));
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bar.comp_ready[half]);
      }
      if (!ok) break;
      if (!wait_all(&bar.acc_done, ucnt & 1)) break;
      tc_fence_after();
      {
        // tcgen05.ld is warp-collective: every lane loads, only real query rows are stored
        __nv_bfloat16* dqr =
            a.dq + w.b * a.dq_sb + (int64_t)(valid ? qi : 0) * a.dq_ss + (int64_t)w.h * a.dq_sh + c_lo;
#pragma unroll 1
        for (int c = 0; c < D / 2; c += 32) {
          float q0[32];
          tmem_ld32f(lane_base + 256 + c_lo + c, q0);
          tmem_ld_wait();
          reg_fence_f<32>(q0);
#pragma unroll
          for (int e = 0; valid && e < 32; e += 8) {
            uint4 pq;
            pq.x = pack_bf16x2(q0[e] * a.scale, q0[e + 1] * a.scale);
            pq.y = pack_bf16x2(q0[e + 2] * a.scale, q0[e + 3] * a.scale);
            pq.z = pack_bf16x2(q0[e + 4] * a.scale, q0[e + 5] * a.scale);
            pq.w = pack_bf16x2(q0[e + 6] * a.scale, q0[e + 7] * a.scale);
            *reinterpret_cast<uint4*>(dqr + c + e) = pq;
          }
          __syncwarp();  // reconverge before the next warp-collective load
        }
      }
      tc_fence_before();
      mbar_arrive(&bar.acc_free);
      gstep += w.n;
      ++ucnt;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kBMmaWarp) {
    __syncwarp();
    tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0 && bar.abort_flag && a.status) atomicOr(a.status, BDEV_TIMEOUT);
}

}  // namespace attn_bwd_kernels
