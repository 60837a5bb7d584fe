/*
 * attn.h - C ABI of the B200 (sm_100a) exact-attention forward library.
 *
 * The library computes exact scaled-dot-product attention forward,
 *     O = softmax(score_mod(scale * Q K^T) + mask) V,
 * tile by tile with an online (running max / running sum) softmax, so the
 * Sq x Skv score matrix never reaches device memory ("A Deep Dive into Flash
 * Attention": sections "Tiling the Computation", "2. Online Softmax",
 * "3. Weighted Sum of Values"). The options are those of flash_attn_func /
 * flash_attn_with_kvcache (FlashAttention overview, "Examples": softmax_scale,
 * causal, window_size, alibi_slopes, cache_seqlens, block_table) and the
 * FlexAttention hooks (attention-gym issue 101 repro: mask_mod q_idx >= kv_idx,
 * create_block_mask with BLOCK_SIZE; "FlexAttention + FlashAttention-4" talk:
 * score mods ALiBi / softcap, masks causal / sliding window, block sparsity).
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    allocates nothing, frees nothing and never synchronises the stream.
 *  - `stream` is a cudaStream_t passed as void*; every launch goes on it.
 *  - Argument checks run on the host before any launch and return a status;
 *    no C++ exception crosses this boundary.
 *  - Kernel-detected problems (a wait that timed out, a page id outside the
 *    cache) are OR-ed into the optional device int `*status` (ATTN_DEV_* bits)
 *    and never trap. The caller reads it when it chooses.
 *  - Inputs are bf16 (raw 16-bit storage), accumulation is fp32, O is bf16,
 *    LSE is fp32 natural-log.
 *  - Element strides are in elements; the head dimension is contiguous. Every
 *    non-unit stride must be a multiple of 8 elements (16 bytes) and every
 *    tensor base 16-byte aligned (a TMA requirement).
 */
#ifndef ATTN_H
#define ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = 1,  /* a pointer, size, stride or option is malformed */
  ATTN_ERR_UNSUPPORTED = 2,  /* well-formed but outside what the kernels handle */
  ATTN_ERR_CUDA = 3,         /* a CUDA runtime / driver call failed */
  ATTN_ERR_WORKSPACE = 4     /* the caller's workspace is too small */
} attn_status;

/* Bits the kernels OR into *status. */
#define ATTN_DEV_TIMEOUT 1   /* a bounded pipeline wait gave up; outputs invalid */
#define ATTN_DEV_BAD_PAGE 2  /* a block_table entry was outside [0, num_pages) */
#define ATTN_DEV_BAD_MASK 8  /* prefill: a caller-written block-mask table had a row_order entry
                                outside [0, n_q_tiles) or a count outside [0, n_kv_tiles); the
                                entry was not followed (default order / clamped count) */
#define ATTN_DEV_BAD_LEN 4   /* decode: a cache_seqlens[b] was negative or above max_seqlen;
                                that sequence was computed over its first max_seqlen keys
                                (none if negative) and its outputs are not the requested ones */

/* Mask kinds (FlexAttention mask_mod equivalents, attention-gym issue 101 and
 * the FA4 talk; flash_attn window_size in the FlashAttention overview).
 * With q_pos = i + q_offset for query i and key position j:
 *   NONE      every key allowed
 *   CAUSAL    j <= q_pos                                   (q_idx >= kv_idx)
 *   WINDOW    (left < 0 || q_pos - j <= left) && (right < 0 || j - q_pos <= right)
 *   DOCUMENT  j <= q_pos && doc[b][i] == doc[b][j]   (packed sequences; Sq == Skv,
 *             q_offset == 0; needs a block mask built from the same spec) */
typedef enum { ATTN_MASK_NONE = 0, ATTN_MASK_CAUSAL = 1, ATTN_MASK_WINDOW = 2, ATTN_MASK_DOCUMENT = 3 } attn_mask_kind;

/* Score modifiers applied to the scaled score s = scale * q.k before masking
 * (FA4 talk, score_mod hooks; flash_attn alibi_slopes and softcapping):
 *   SOFTCAP   s -> softcap * tanh(s / softcap)
 *   ALIBI     s -> s + slope[b][h] * (j - q_pos)                                */
/* Score modifiers (FlexAttention score_mod hooks; flash_attn_func's softcap
 * and alibi_slopes). ATTN_MOD_RELU is the talk's activation wrapper: the
 * softmax normalisation is undone and each allowed scaled score passes
 * through ReLU, O = sum_j max(scale q.k_j, 0) v_j, with ln(sum_j of those
 * weights) in the LSE slot (-inf when they sum to 0); attn_fwd only. */
typedef enum { ATTN_MOD_NONE = 0, ATTN_MOD_SOFTCAP = 1, ATTN_MOD_ALIBI = 2, ATTN_MOD_RELU = 3 } attn_mod_kind;

typedef struct {
  attn_mask_kind kind;
  int window_left;        /* WINDOW: keys at most this far behind; -1 = unbounded */
  int window_right;       /* WINDOW: keys at most this far ahead;  -1 = unbounded */
  int q_offset;           /* position of query 0 on the key axis (CAUSAL / WINDOW) */
  const int32_t *doc_id;  /* DOCUMENT: device int32 document id per position, 16-byte aligned:
                             row b (batch b) starts at doc_id + b * doc_batch_stride */
  int64_t doc_batch_stride; /* elements between the rows of doc_id (a multiple of 4); 0 = one
                               [S] row shared by every batch */
} attn_mask_spec;

/* Block mask (FlexAttention create_block_mask(mask_mod, B, H, Q_LEN, KV_LEN,
 * BLOCK_SIZE) equivalent, attention-gym issue 101): per (batch, head, q-tile,
 * kv-tile) class 0 = empty (skipped), 1 = partial (mask evaluated per
 * element), 2 = full (no mask work), and per (batch, head, q-tile) the
 * ascending kv-tile lists of partial and full tiles. Bm / Hm are the batch and
 * head extents of the tables: 1 means one slice shared by every batch / head,
 * otherwise they equal the B / Hq of the forward call (slice (b, h) serves
 * batch b, query head h). All arrays live inside one caller-owned device
 * buffer laid out by attn_block_mask_layout; a caller may also fill the
 * tables itself (for example per-head block-sparse patterns over MASK_NONE),
 * as long as every list is ascending and consistent with cls. */
typedef struct {
  int Bm, Hm;
  int Sq, Skv, blk_q, blk_kv, n_q_tiles, n_kv_tiles;
  uint8_t *cls;       /* [Bm][Hm][n_q_tiles][n_kv_tiles] */
  int32_t *part_cnt;  /* [Bm][Hm][n_q_tiles] */
  int32_t *part_idx;  /* [Bm][Hm][n_q_tiles][n_kv_tiles], first part_cnt entries of a row valid */
  int32_t *full_cnt;  /* [Bm][Hm][n_q_tiles] */
  int32_t *full_idx;  /* [Bm][Hm][n_q_tiles][n_kv_tiles], first full_cnt entries of a row valid */
  /* Work order (scheduling only, never changes a result): [Bm][n_q_tiles], the
   * q-tiles of batch slice b (head slice 0) by decreasing number of visited
   * kv tiles (part_cnt + full_cnt), ties by index. NULL = last q-tile first.
   * attn_build_block_mask fills it; a caller filling the tables itself may
   * set it to NULL or write any permutation. */
  int32_t *row_order;
  /* DOCUMENT masks (filled by attn_build_block_mask from the document rows):
   * doc_sorted[b] = 1 when the ids of row b never decrease, and then
   * doc_start[b][i] is the first position of the run of equal ids holding i,
   * so that key j <= i is allowed iff j >= doc_start[b][i] (each document is
   * one run). Rows with doc_sorted 0 are masked by comparing ids. */
  int32_t *doc_start; /* [Bm][Sq] */
  int32_t *doc_sorted;/* [Bm] */
} attn_block_mask;

/* Bytes of device memory a block mask for these sizes needs (0 if invalid). */
size_t attn_block_mask_bytes(int Bm, int Hm, int Sq, int Skv, int blk_q, int blk_kv);

/* Carves the tables out of `buf` (device, >= attn_block_mask_bytes, 16-byte
 * aligned) and fills `out`. Host-only pointer arithmetic; nothing is launched. */
attn_status attn_block_mask_layout(void *buf, size_t buf_bytes, int Bm, int Hm, int Sq, int Skv, int blk_q,
                                   int blk_kv, attn_block_mask *out);

/* Classifies every tile of the mask on the device by evaluating the mask on
 * each in-range (q, kv) pair (out-of-range positions of ragged edge tiles do
 * not count) and writes the class tables and both ascending index lists of
 * every (batch, head) slice. A DOCUMENT mask reads document row b for slice
 * b (row 0 for every slice when doc_batch_stride is 0); the mask kinds do not
 * depend on the head, so the Hm slices of a batch are equal. Any mask kind is
 * accepted; blk_q and blk_kv must be multiples of 16. */
attn_status attn_build_block_mask(const attn_mask_spec *spec, const attn_block_mask *out, void *stream);

typedef struct {
  const void *q;              /* bf16 [B][Sq][Hq][D] via q_stride */
  const void *k;              /* bf16 [B][Skv][Hkv][D] via k_stride */
  const void *v;              /* bf16 [B][Skv][Hkv][D] via v_stride */
  void *o;                    /* bf16 [B][Sq][Hq][D] via o_stride (output) */
  float *lse;                 /* fp32 [B][Hq][Sq] contiguous (output); may be NULL */
  int64_t q_stride[3];        /* element strides of batch, sequence, head */
  int64_t k_stride[3];
  int64_t v_stride[3];
  int64_t o_stride[3];
  int B, Hq, Hkv, Sq, Skv, D; /* Hq % Hkv == 0 (GQA/MQA without repeat_kv); D in {64, 128} */
  float scale;                /* softmax_scale; <= 0 selects 1/sqrt(D) */
  attn_mask_spec mask;
  const attn_block_mask *block_mask; /* optional for NONE/CAUSAL/WINDOW, required for
                                        DOCUMENT; 128 x 128 tiles for (Sq, Skv), Bm in {1, B},
                                        Hm in {1, Hq} */
  attn_mod_kind mod;
  float softcap;              /* SOFTCAP: cap > 0 */
  const float *alibi_slopes;  /* ALIBI: device fp32 [Hq] or [B][Hq] */
  int alibi_batch_stride;     /* 0 for [Hq], Hq for [B][Hq] */
  int *status;                /* optional device int, ATTN_DEV_* bits OR-ed in */
} attn_fwd_params;

/* Prefill / full-sequence forward: O and LSE for every query row. Empty
 * tiles are skipped, full tiles do no mask work. Rows with no allowed key get
 * O = 0 and LSE = -inf. Sq == 0 or B == 0 launches nothing. */
attn_status attn_fwd(const attn_fwd_params *p, void *stream);

typedef struct {
  const void *q;              /* bf16 [B][Hq][D] (one new token per sequence) via q_stride */
  int64_t q_stride[2];        /* element strides of batch, head */
  const void *k_cache;        /* bf16 [num_pages][page_size][Hkv][D] via cache_stride */
  const void *v_cache;        /* same shape and strides as k_cache */
  int64_t cache_stride[3];    /* element strides of page, slot, head */
  const int32_t *block_table; /* int32 [B][block_table_stride]: logical page -> physical page */
  int block_table_stride;     /* >= max pages any sequence uses */
  const int32_t *cache_seqlens; /* int32 [B]: keys of sequence b are its first cache_seqlens[b] tokens */
  int B, Hq, Hkv, D, page_size, num_pages;
  int max_seqlen;             /* upper bound on every cache_seqlens[b] (sizes the splits); a
                                 larger or negative length is clamped to [0, max_seqlen] and
                                 reported as ATTN_DEV_BAD_LEN in *status */
  float scale;                /* <= 0 selects 1/sqrt(D) */
  attn_mod_kind mod;          /* the query sits at position cache_seqlens[b] - 1 */
  float softcap;
  const float *alibi_slopes;
  int alibi_batch_stride;
  int num_splits;             /* key-axis splits per sequence; 0 = choose automatically */
  void *o;                    /* bf16 [B][Hq][D] via o_stride (output) */
  int64_t o_stride[2];
  float *lse;                 /* fp32 [B][Hq] contiguous (output); may be NULL */
  int *status;                /* optional device int, ATTN_DEV_* bits */
  /* Several new tokens per sequence (flash_attn_with_kvcache with q of
   * seqlen > 1): q and o are [B][q_len][Hq][D], token i at q_token_stride /
   * o_token_stride elements from token 0; lse is [B][q_len][Hq] contiguous.
   * The q_len tokens of a sequence sit at its last q_len key positions, and
   * their q_len x g heads share one 128-row MMA tile: q_len * (Hq / Hkv)
   * <= 128. 0 means 1 (the fields above alone describe the call). */
  int q_len;
  int64_t q_token_stride, o_token_stride;
  int causal;                 /* q_len > 1: token i sees the first cache_seqlens[b] - (q_len - 1 - i) keys */
  /* block_table == NULL selects a contiguous cache: k_cache / v_cache are
   * [num_pages = cache rows][page_size = positions][Hkv][D] and sequence b
   * reads row cache_batch_idx[b] (row b when cache_batch_idx is NULL);
   * page_size >= max_seqlen, no divisibility rule. */
  const int32_t *cache_batch_idx;
} attn_decode_params;

/* Number of splits attn_decode uses for these sizes (resolves num_splits = 0).
 * An explicit num_splits is clamped to the number of 128-key tiles of
 * max_seqlen. Automatic: the count minimising waves of CTAs x (tiles per split
 * + a fixed per-unit cost of ten tiles), fewer splits on ties, so one full
 * wave of (sequence, KV head, split) units is preferred when it fits. */
int attn_decode_num_splits(int B, int Hq, int Hkv, int max_seqlen, int num_splits);

/* Workspace bytes attn_decode needs: one fp32 partial O row and LSE per
 * (sequence, query head, split); with q_len new tokens pass Hq * q_len. */
size_t attn_decode_workspace_bytes(int B, int Hq, int D, int num_splits);

/* Split-KV decode over a paged KV cache (flash_attn_with_kvcache with
 * block_table and cache_seqlens, FlashAttention overview, "Examples"): each
 * (sequence, KV head, split) runs the online softmax over its share of the
 * keys with all query heads of the group as the MMA rows and writes a partial
 * (O_i, LSE_i); a second kernel combines them, LSE = ln sum_i exp(LSE_i) and
 * O = sum_i exp(LSE_i - LSE) O_i. page_size must be a multiple of 16 that
 * divides 128 or is a multiple of 128. `workspace` is caller-owned device
 * memory of at least attn_decode_workspace_bytes(B, Hq, D, splits). */
attn_status attn_decode(const attn_decode_params *p, void *workspace, size_t workspace_bytes, void *stream);

/* The combine step on its own: merges n_splits partial results per row.
 * o_parts fp32 [rows][n_splits][D] (normalised partial outputs), lse_parts fp32
 * [rows][n_splits] (natural log, -inf = empty part); writes o bf16
 * [rows][D] with row stride o_row_stride (elements) and lse fp32 [rows]
 * (may be NULL). D in {64, 128}. */
attn_status attn_lse_combine(const float *o_parts, const float *lse_parts, int rows, int n_splits, int D, void *o,
                             int64_t o_row_stride, float *lse, void *stream);

/* attn_decode without a caller-provided workspace. The paper has no
 * counterpart: this exists for callers that are not allowed to allocate
 * device memory (a plugin that is handed only its inputs and outputs by an
 * engine that plans all device memory up front, or a latency-critical loop
 * that cannot risk cudaMalloc's device-wide synchronisation). The split
 * partials live in a fixed array inside the library, ATTN_DECODE_NOALLOC_MAX_BYTES
 * per device, held by every GPU that loads the library until exit.
 *  - Same parameters and results as attn_decode.
 *  - Returns ATTN_ERR_WORKSPACE, launching nothing, when the call's partials
 *    (attn_decode_workspace_bytes for its B, Hq, D and split count) exceed the
 *    maximum; pass a smaller num_splits or batch, or use attn_decode.
 *  - The first call on a device looks up the array's device address (and may
 *    load the device code); make it before any stream capture on that device.
 *  - All calls on a device share the array and leave their partials in it;
 *    nothing needs clearing, but calls that overlap on the GPU race, so keep
 *    them ordered on one stream.
 *  - Allocates and frees nothing. */
#define ATTN_DECODE_NOALLOC_MAX_BYTES (32u * 1024u * 1024u)
attn_status attn_decode_noalloc(const attn_decode_params *p, void *stream);

/* In-place kv-cache update with rotary embedding (FlashAttention overview,
 * "Examples": flash_attn_with_kvcache's k, v, rotary_cos, rotary_sin,
 * rotary_interleaved, cache_batch_idx and block_table arguments). For every
 * sequence b and new token i (position p = cache_seqlens[b] + i):
 *   - k_new[b][i] rotated by the angles at p and v_new[b][i] are written to
 *     the cache at position p (paged: page block_table[b][p / page_size], row
 *     p % page_size; contiguous: row cache_batch_idx[b] or b, position p);
 *   - q[b][i] rotated at p is written to q_out (q_out may equal q);
 *   - seqlens_out[b] = cache_seqlens[b] + Snew when seqlens_out is given.
 * Rotation: pair j of a head vector is (x[2j], x[2j+1]) when interleaved,
 * else (x[j], x[j + rotary_dim / 2]), turned by cos/sin[p][j] in fp32 and
 * rounded to bf16; dims past rotary_dim are copied. rotary_cos == NULL
 * skips rotation (q_out then receives a copy of q, if both are given).
 * Kernel-detected errors, OR-ed into *status, skip the row: a page id
 * outside [0, num_pages) or a logical page past block_table_stride
 * (ATTN_DEV_BAD_PAGE), a position past the cache or the rotary table
 * (ATTN_DEV_BAD_LEN). One HBM-bound kernel; nothing is allocated. */
typedef struct {
  const void *q;                  /* bf16 [B][Snew][Hq][D] via q_stride, or NULL */
  int64_t q_stride[3];
  void *q_out;                    /* bf16, shaped like q, via q_out_stride */
  int64_t q_out_stride[3];
  const void *k_new, *v_new;      /* bf16 [B][Snew][Hkv][D] via the strides, or both NULL */
  int64_t k_new_stride[3], v_new_stride[3];
  void *k_cache, *v_cache;        /* bf16, same layout: paged [pages][page_size][Hkv][D] or contiguous */
  int64_t cache_stride[3];        /* element strides of page (row), slot (position), head */
  const int32_t *block_table;     /* int32 [B][block_table_stride], or NULL for a contiguous cache */
  int block_table_stride;
  const int32_t *cache_batch_idx; /* contiguous cache: int32 [B] cache row of each sequence, or NULL */
  const int32_t *cache_seqlens;   /* int32 [B]: tokens in the cache before the update */
  int32_t *seqlens_out;           /* int32 [B] or NULL */
  int B, Snew, Hq, Hkv, D, page_size, num_pages;
  const float *rotary_cos, *rotary_sin; /* fp32 [rotary_positions][rotary_dim / 2], or NULL */
  int rotary_dim;                 /* multiple of 16, <= D */
  int rotary_positions;
  int rotary_interleaved;
  int *status;                    /* optional device int */
} attn_kvcache_update_params;

attn_status attn_kvcache_update(const attn_kvcache_update_params *p, void *stream);

/* Backward of attn_fwd (FlashAttention overview, "Examples": the backward
 * pass of flash_attn_func and its `deterministic` option): dQ, dK, dV for the
 * upstream gradient dO, from Q, K, V, the forward's O and LSE. With
 * P = exp(scale * Q K^T - LSE) over the allowed pairs:
 *   dV = P^T dO,  dS = P o (dO V^T - rowsum(dO o O)),  dQ = scale dS K,  dK = scale dS^T Q,
 * with dK and dV summed over the query heads of each KV head (GQA/MQA).
 * Kernels: a row reduction for rowsum(dO o O) into the workspace (whose
 * last block also writes the dK/dV work plan there), one tcgen05 kernel over
 * pieces of key tiles (dK, dV; a key tile with more steps than a cap set
 * from the work per SM is cut into pieces whose fp32 partials a reduction
 * kernel sums in piece order) and one over query tiles (dQ). Every output
 * element is accumulated in a fixed order with no atomics, so results are
 * bit-identical from run to run on a device whatever `deterministic` says
 * (the flag is accepted for interface compatibility).
 * Supported: masks NONE / CAUSAL / WINDOW, no score mod, D in {64, 128};
 * anything else returns ATTN_ERR_UNSUPPORTED. Layout rules as for attn_fwd;
 * `workspace` is caller-owned device memory, 16-byte aligned, of at least
 * attn_bwd_workspace_bytes(p) bytes for the same parameters on the same
 * device (the plan depends on the device's SM count). Sq == 0 or B == 0
 * launches nothing; Skv == 0 gives dQ = 0 (dK, dV are empty). */
typedef struct {
  const void *q, *k, *v, *o, *dout;  /* bf16 [B][S][H][D] via the strides below */
  const float *lse;                  /* fp32 [B][Hq][Sq] contiguous, natural log, from attn_fwd */
  void *dq, *dk, *dv;                /* bf16 outputs, shaped like q, k, v */
  int64_t q_stride[3], k_stride[3], v_stride[3], o_stride[3], do_stride[3];
  int64_t dq_stride[3], dk_stride[3], dv_stride[3];
  int B, Hq, Hkv, Sq, Skv, D;
  float scale;                       /* <= 0 selects 1/sqrt(D) */
  attn_mask_spec mask;               /* NONE, CAUSAL or WINDOW */
  int deterministic;
  int *status;                       /* optional device int, ATTN_DEV_* bits */
} attn_bwd_params;

/* Workspace bytes attn_bwd needs for these parameters on the current
 * device: the delta rows, the dK/dV plan and the partials of split key
 * tiles. 0 when the parameters are invalid or unsupported. */
size_t attn_bwd_workspace_bytes(const attn_bwd_params *p);
attn_status attn_bwd(const attn_bwd_params *p, void *workspace, size_t workspace_bytes, void *stream);

/* Failure-detection self-test (no counterpart on the pages). Launches one
 * warp that waits, with the bounded wait every pipeline barrier of these
 * kernels uses, on a barrier nothing arrives on. After the wait's limit
 * (about one second of SM clock) the kernel ORs ATTN_DEV_TIMEOUT into
 * *status and exits normally; the context stays usable.
 *  - status: device int (caller-owned), read by the caller after the stream
 *    is synchronised.
 *  - Returns ATTN_ERR_INVALID_ARG for a NULL status, ATTN_ERR_CUDA if the
 *    launch fails, ATTN_OK otherwise. Asynchronous on the given stream. */
attn_status attn_selftest_wait_timeout(int *status, void *stream);

const char *attn_status_str(attn_status s);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_H */
