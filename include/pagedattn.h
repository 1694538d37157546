/*
 * pagedattn.h - C ABI of a B200 (sm_100a) attention library over a paged KV cache.
 *
 * The library computes FlashAttention-style tiled, online-softmax attention
 * over a two-level KV cache: a table maps (request, position) to a token slot
 * ("req_to_token") and per-layer pools map a slot to that layer's K and V rows
 * ("token_to_kv_pool")  ["Implement Flash Attention Back End in SGLang -
 * Basics and KV Cache", KV-cache passage; "Flash Attention Backend in SGLang:
 * Grundlagen und KV Cache optimal nutzen", req_to_token / token_to_kv_pool
 * paragraph].  With a page size P > 1 the table holds page numbers
 * ["PagedAttention: 优化 KV Cache 的管理和利用率", section 2, 工作原理]:
 *
 *     slot(r, j) = page_table[r * pt_pitch + j / P] * P + j % P
 *
 * Two forward modes are provided, DECODE (one query token per request) and
 * EXTEND (new tokens attending causally to a cached prefix and to themselves)
 * [forward modes in the same two SGLang pages], plus the 8-bit "Sage" decode
 * ["FlashInfer PrimTS, Sage Attention 도입으로 8비트 양자화 및 성능 최적화 달성",
 * section "코드 분석" items 1 and 4].
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Pointers prefixed d_ or naming device tensors are DEVICE pointers; struct
 *   pointers (pa_plan_params*, size_t*) are HOST pointers.  The caller owns
 *   every buffer, including the plan workspace; the library allocates and
 *   frees nothing and keeps no pointer between calls.
 * - bf16 tensors are passed as raw 16-bit bit patterns (uint16_t); E4M3
 *   tensors as raw bytes (uint8_t).
 * - Layouts (row-major, innermost last):
 *     K/V pools       [num_slots][Hkv][D]        per layer
 *     page_table      int32 [B][pt_pitch]        page (or, for P = 1, slot) ids
 *     DECODE Q, O     [B][Hq][D];  lse [B][Hq]
 *     EXTEND Q, O     [sum_r n_r][Hq][D];  lse [sum_r n_r][Hq]
 *   Query head h reads KV head h / (Hq / Hkv).
 * - Every call only enqueues work on `stream` and never synchronises the host
 *   (except pa_read_device_error), so a plan followed by per-layer calls can
 *   be captured in a CUDA graph.  Launch geometry depends only on the host
 *   parameters, never on device data.
 * - Functions return a status and never throw.  Scale values and table
 *   contents are not validated on the host; a slot or page id outside the pool
 *   is skipped (its row reads as zero) and recorded in the workspace's device
 *   error word, which pa_read_device_error reports as PA_ERR_DEVICE_INDEX.
 * - Head dimension D must be 128; the page size must be a power of two
 *   <= 256; Hq / Hkv must be 1, 2, 4 or 8.
 */
#ifndef PAGEDATTN_H
#define PAGEDATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* pa_stream_t;

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID = 1,       /* NULL where required, inconsistent sizes, misaligned buffer,
                               an input the mode does not use passed non-NULL, bad plan mode */
  PA_ERR_UNSUPPORTED = 2,   /* head_dim != 128, page size not a power of two <= 256,
                               Hq / Hkv not in {1,2,4,8}, Sage shared-memory budget exceeded,
                               Sage page size other than 64 */
  PA_ERR_ARCH = 3,          /* the current device is not sm_100 (B200) */
  PA_ERR_WORKSPACE = 4,     /* workspace too small, or a run call's mode differs from the plan's */
  PA_ERR_CUDA = 5,          /* a CUDA runtime call or kernel launch failed */
  PA_ERR_DEVICE_INDEX = 6   /* (pa_read_device_error only) a kernel met an out-of-range
                               slot/page id or sequence length, or gave up a bounded wait */
} pa_status;

typedef enum {
  PA_MODE_DECODE = 0,       /* bf16 split-KV decode + log-sum-exp merge */
  PA_MODE_EXTEND = 1,       /* bf16 causal extend over a cached prefix (tcgen05 / TMEM) */
  PA_MODE_SAGE_DECODE = 2,  /* INT8 Q/K, E4M3 P and V, per-block scales, bf16 output */
  PA_MODE_SAGE_SPARSE = 3   /* SAGE_DECODE over the selected 64-key blocks of each request */
} pa_mode;

/*
 * Plan-time parameters: fixed per batch, shared by every layer's run call
 * ("the recipe is fixed at plan time, the scales are given at every run",
 * "FlashInfer PrimTS, Sage Attention ..." section "코드 분석" items 1 and 5).
 */
typedef struct {
  int32_t mode;          /* pa_mode */
  int32_t batch;         /* B, number of requests, 1 .. 8192 */
  int32_t hq;            /* query heads */
  int32_t hkv;           /* KV heads; hq % hkv == 0 and hq / hkv in {1, 2, 4, 8} */
  int32_t head_dim;      /* D, must be 128 */
  int32_t page_size;     /* P: power of two, 1 .. 256 (SAGE: == sage_k_block) */
  int32_t max_kv_len;    /* upper bound on every seq_lens[r]; longer lengths are clamped and flagged */
  int32_t max_q_tokens;  /* EXTEND: upper bound on sum of new tokens (sizes the grid); else 0 */
  int32_t num_sms;       /* SMs the plan schedules for; 0 = query the current device */
  int32_t max_splits;    /* DECODE and SAGE: 0 (the flat partition needs no cap); EXTEND: 0 or 1 */
  int32_t sage_k_block;  /* SAGE: keys per sfK block, must be 64; else 0 */
  int32_t reserved;      /* must be 0 */
} pa_plan_params;

/*
 * Workspace bytes needed by attn_plan and the run calls for `params`
 * (header, per-request arrays, the work list and, for DECODE, the split
 * partials).  Writes *bytes; returns PA_ERR_INVALID / PA_ERR_UNSUPPORTED for
 * parameters that attn_plan would reject.  Host only, no CUDA work except a
 * device-attribute query when num_sms == 0.
 */
pa_status pa_plan_workspace_size(const pa_plan_params* params, size_t* bytes);

/*
 * attn_plan - build the per-batch scheduling metadata once, for reuse by every
 * layer ["SGLang의 FA3 디코드 최적화: get_scheduler_metadata 도입", 코드 분석
 * items 1-3 and 왜 이게 좋은가 item 1: the metadata depends only on the
 * sequence lengths and the optional cumulative query lengths].
 *
 * d_seq_lens     int32 [B], device: total KV length L_r of each request (for
 *                EXTEND, prefix plus new tokens).
 * d_cu_seqlens_q int32 [B+1], device: EXTEND only (exclusive prefix sums of
 *                the new-token counts); must be NULL for the other modes.
 * d_ws           device workspace of ws_bytes >= pa_plan_workspace_size().
 *
 * One single-CTA kernel computes, from the lengths alone (integer arithmetic):
 *   DECODE and SAGE_DECODE: a flat, balanced partition of the requests' units
 *     over CTA slots.  A unit is U keys: U = T = max(64, P) for DECODE, U = 32
 *     for SAGE_DECODE; units_r = ceil(L_r / U).  A work item covers HG = the
 *     largest of 8, 4, 2, 1 dividing Hkv KV heads, groups = Hkv / HG, and
 *     C = max(1, floor(num_sms * 2 / groups)) CTA slots (two slots per SM),
 *     g_r = sum of the units of the requests before r, total = sum units_r,
 *     per = max(1, ceil(total / C)), used = ceil(total / per).  Slot c takes the
 *     concatenated units [c per, (c+1) per); each maximal piece of that range
 *     within one request is an item (r, s, U u0, min(U u1, L_r)), u0/u1 relative
 *     to g_r and s the piece's index within request r; an empty request is one
 *     item (r, 0, 0, 0) of slot min(floor(g_r / per), max(used - 1, 0)).  Items
 *     are listed r-major (which is also slot order, no sort) and slot_first[c],
 *     c = 0 .. C, is the first item of slot c or later (num_items if none).  A
 *     run CTA walks every item of its slot, so every slot streams at most per
 *     units and the slots finish together; max_splits must be 0.
 *   EXTEND: query tiles of 128 new tokens; tile t of request r covers new
 *     tokens [128 t, min(128 t + 128, n_r)) and reads key tiles
 *     0 .. ceil((p_r + q_end) / 128) - 1, p_r = L_r - n_r.  Items are ordered
 *     by that key-tile count descending, ties by (request, tile) order, so the
 *     in-order block dispatch of the run kernel schedules the longest work first.
 *   SAGE_SPARSE: the SAGE_DECODE partition over the units of each request's selected
 *     blocks (attn_plan_sage_sparse): sel_r = the selected blocks in ascending order, a
 *     selected block holds 2 units except a last block of L_r - 64 b <= 32 keys (1 unit);
 *     items are (r, s, u0, u1) in unit indices of request r, unit u being keys
 *     64 sel_r[u / 2] + 32 (u % 2) onward (at most 32, not past L_r).
 * At most C + B items (DECODE, SAGE) or ceil(max_q_tokens / 128) + B (EXTEND).
 *
 * Workspace layout (for introspection; all int32, offsets in bytes):
 *   [0, 64)   header: magic 0x4C504150, mode, batch, hq, hkv, head_dim,
 *             page_size, num_items, max_items, tile, chunk_tiles, error word,
 *             num_sms, max_splits, slots (DECODE, SAGE: C, else 0), reserved
 *   then      req_splits[B] (items of request r), req_base[B+1] (exclusive
 *             prefix sum of req_splits), req_len[B] (L_r as used), req_aux[B]
 *             (DECODE, SAGE: g_r; EXTEND: cu_seqlens_q[r]),
 *             req_prefix[B] (EXTEND: p_r), padded to 16 B, then the items
 *             int32x4 [max_items] = {r, split, begin, end} in execution order,
 *             256-byte aligned, then (DECODE, SAGE) slot_first int32 [C + 1], 256-byte
 *             aligned, then (SAGE_SPARSE) sel_base int32 [B + 1] and sel_block int32
 *             [B * ceil(max_kv_len / 64)], each 256-byte aligned, then (DECODE,
 *             SAGE) fp32 partial outputs
 *             [max_items][Hq][D] and partial LSEs (DECODE: log2 units; SAGE:
 *             the split's row sum l) [max_items][Hq], then (SAGE) the split
 *             maxima fp32 [max_items][Hq] and the score rows fp32
 *             [B][Hq][max(max_kv_len, 64) rounded up to 64], each 256-byte
 *             aligned.
 *             The partial of split s of request r, head h, sits at row
 *             (req_base[r] + s) * Hq + h.
 * Lengths < 0 or > max_kv_len are clamped to [0, max_kv_len] and set the
 * error word.  Returns PA_ERR_ARCH off sm_100, PA_ERR_WORKSPACE if ws_bytes
 * is short, PA_ERR_INVALID for NULL pointers or a cu_seqlens_q that does not
 * match the mode.
 */
pa_status attn_plan(const pa_plan_params* params, const int32_t* d_seq_lens,
                    const int32_t* d_cu_seqlens_q, void* d_ws, size_t ws_bytes,
                    pa_stream_t stream);

/*
 * attn_plan_sage_sparse - the plan of a block-sparse Sage decode (mode PA_MODE_SAGE_SPARSE):
 * Sage attention runs in the dense and block-sparse modes ("FlashInfer PrimTS, Sage
 * Attention ...", README), and, as for the dense plan, the sparsity pattern is fixed when
 * the plan is made.  The reading taken for decode: one mask per (request, logical 64-key
 * block), shared by all heads; request r attends to the keys of its selected blocks only,
 * and the Sage formula (row max and row sum included) runs over that subset.
 *
 * d_block_mask   uint8 [B][mask_pitch], device: nonzero selects block b of request r
 *                (entries at b >= ceil(L_r / 64) are ignored); mask_pitch >=
 *                ceil(max_kv_len / 64).
 * The partition (algorithm at attn_plan, SAGE_SPARSE) runs over the selected blocks'
 * 32-key units, so every CTA slot streams the same number of selected keys; the workspace
 * holds the selected blocks of each request (sel_base, sel_block).  A request with no
 * selected block gives O = v_mean.  Other arguments and errors as for attn_plan.
 */
pa_status attn_plan_sage_sparse(const pa_plan_params* params, const int32_t* d_seq_lens,
                                const uint8_t* d_block_mask, int64_t mask_pitch, void* d_ws, size_t ws_bytes,
                                pa_stream_t stream);

/*
 * attn_decode_paged - bf16 DECODE over the paged cache for one layer.
 * For each request r and query head h:  s_j = sm_scale * q . K_j,
 * O = sum_j softmax(s)_j V_j over j in [0, L_r), lse = log sum_j exp(s_j)
 * ["FlashAttention: 优化计算过程中的临时显存占用", section 1 (the standard
 * definition) and section 2 (tiling reaches it without the N x N matrix)].
 * Each (request, KV head, split) CTA gathers its K/V rows with 16-byte
 * copies through the slot table, packs the Hq / Hkv query heads of the KV head
 * so each row is read once, and keeps a running max / sum; requests split
 * into several key ranges are combined by a log-sum-exp merge kernel.
 *
 * params, d_ws    the plan (mode PA_MODE_DECODE) built by attn_plan.
 * d_q             bf16 [B][Hq][D];  d_k_pool, d_v_pool bf16 [num_slots][Hkv][D].
 * d_page_table    int32 [B][pt_pitch] (pt_pitch >= ceil(max_kv_len / P)).
 * d_out           bf16 [B][Hq][D];  d_lse_out fp32 [B][Hq] natural log, or NULL.
 * All device pointers 16-byte aligned.  Empty requests give O = 0, lse = -inf.
 */
pa_status attn_decode_paged(const pa_plan_params* params, const void* d_ws, size_t ws_bytes,
                            const uint16_t* d_q, const uint16_t* d_k_pool,
                            const uint16_t* d_v_pool, int64_t num_slots,
                            const int32_t* d_page_table, int64_t pt_pitch, float sm_scale,
                            uint16_t* d_out, float* d_lse_out, pa_stream_t stream);

/*
 * attn_decode_paged_fp8 - DECODE over an FP8 KV cache for one layer.  The FlashAttention
 * backend lists FP8 among its features ("Implement Flash Attention Back End in SGLang -
 * Basics and KV Cache", feature list); the operation is the standard decode of
 * attn_decode_paged on the dequantised cache
 *     K = k_scale * E4M3(K8),  V = v_scale * E4M3(V8)     (one scale per pool),
 *     O = softmax(sm_scale * q K^T) V,  lse = log sum_j exp(sm_scale q . K_j).
 * Same plan (mode PA_MODE_DECODE), work list, split partials and merge as the bf16 decode;
 * one CTA covers HG = the largest of 8, 4, 2, 1 dividing Hkv heads (1 KB runs per slot at
 * Hkv = 8).  The tensor cores run in f16 (E4M3 converts to f16 exactly), so |q| must stay
 * below 65504; q values below 2^-24 flush to zero.  Scales are not checked.
 *
 * d_q             bf16 [B][Hq][D];  d_k8_pool, d_v8_pool E4M3 bytes [num_slots][Hkv][D].
 * Everything else as for attn_decode_paged (any page size 1 .. 256).
 */
pa_status attn_decode_paged_fp8(const pa_plan_params* params, const void* d_ws, size_t ws_bytes,
                                const uint16_t* d_q, const uint8_t* d_k8_pool, const uint8_t* d_v8_pool,
                                float k_scale, float v_scale, int64_t num_slots,
                                const int32_t* d_page_table, int64_t pt_pitch, float sm_scale,
                                uint16_t* d_out, float* d_lse_out, pa_stream_t stream);

/*
 * attn_extend_paged - bf16 causal EXTEND for one layer.  New token i of
 * request r (row cu_seqlens_q[r] + i of Q) sits at absolute position p_r + i
 * and attends to keys j <= p_r + i, whose K/V (prefix and new tokens alike)
 * are already in the pool.  O = softmax(sm_scale Q K^T + mask) V.
 * Query tiles of 128 rows per head; QK^T and PV run on the tcgen05 tensor
 * cores with TMEM accumulators; key tiles above the diagonal are skipped.
 * Key pages of 8 or more slots arrive by TMA (one box per page); smaller pages,
 * down to the slot-granular page size 1 where the table is req_to_token itself,
 * are gathered slot by slot with 16-byte copies.  With 4 or 8 query heads per KV
 * head, a pair of CTAs serves four heads and the tensor cores' two-SM form
 * shares every K/V tile between them (each SM loads half of it).
 *
 * params, d_ws    the plan (mode PA_MODE_EXTEND); any page size 1 .. 256.
 * d_q, d_out      bf16 [sum n][Hq][D];  d_lse_out fp32 [sum n][Hq] or NULL.
 * Pools and table as for attn_decode_paged; num_slots < 2^31.
 */
pa_status attn_extend_paged(const pa_plan_params* params, const void* d_ws, size_t ws_bytes,
                            const uint16_t* d_q, const uint16_t* d_k_pool,
                            const uint16_t* d_v_pool, int64_t num_slots,
                            const int32_t* d_page_table, int64_t pt_pitch, float sm_scale,
                            uint16_t* d_out, float* d_lse_out, pa_stream_t stream);

/*
 * attn_decode_paged_sage - 8-bit Sage DECODE for one layer
 * ["FlashInfer PrimTS, Sage Attention ...", 코드 분석 item 1, README formula]:
 *   S_j  = sfQ[r][h] * sfK[slot_j / 64][h_kv] * (Q8 . K8_j)      (exact int dot)
 *   m    = max_j S_j over the whole row,  p_j = exp(S_j - m),  l = sum_j p_j
 *   P8_j = E4M3(448 p_j)                (round to nearest even, saturating)
 *   O[d] = sfV[h_kv][d] * (sum_j P8_j V8_j[d]) / (448 l) + v_mean[h_kv][d]
 * The scales enter before the max and the exponential and sfV is applied in
 * the epilogue (same page, item 4).  S is formed in float32 as
 * (sfQ * sfK) * float(dot).  There is no separate softmax scale: fold it into
 * sfQ.  Scales must be finite and positive and are NOT checked (same page,
 * item 1).
 *
 * params, d_ws    the plan (mode PA_MODE_SAGE_DECODE, or PA_MODE_SAGE_SPARSE from
 *                 attn_plan_sage_sparse; sage_k_block = 64 = page_size).
 * d_q8 int8 [B][Hq][D];  d_sf_q fp32 [B][Hq].
 * d_k8_pool int8, d_v8_pool E4M3 bytes, both [num_slots][Hkv][D].
 * d_sf_k fp32 [num_slots / 64][Hkv];  d_sf_v fp32 [Hkv][D];
 * d_v_mean fp32 [Hkv][D] or NULL (then 0).   d_out bf16 [B][Hq][D].
 * d_sf_k, d_sf_v and d_v_mean 16-byte aligned, like the 8-bit tensors and d_out.
 * Three kernels over the plan's CTA slots: a score pass writes S of every key
 * and query head to the workspace's score rows and each item's per-head
 * maximum; a value pass takes m as the maximum of the request's item maxima
 * (the exact row max), forms P8 from the stored S and accumulates P8 . V8 per
 * item; a merge sums the items (no rescale: all used the same m).  Rows of
 * any length up to max_kv_len are supported; the workspace grows with
 * B * Hq * max_kv_len * 4 bytes of score rows.
 * Empty requests give O = v_mean.
 */
pa_status attn_decode_paged_sage(const pa_plan_params* params, const void* d_ws, size_t ws_bytes,
                                 const int8_t* d_q8, const float* d_sf_q,
                                 const int8_t* d_k8_pool, const uint8_t* d_v8_pool,
                                 const float* d_sf_k, const float* d_sf_v, const float* d_v_mean,
                                 int64_t num_slots, const int32_t* d_page_table, int64_t pt_pitch,
                                 uint16_t* d_out, pa_stream_t stream);

/*
 * attn_extend_paged_sage - 8-bit Sage EXTEND (prefill over a cached prefix) for one layer:
 * the Sage formula of attn_decode_paged_sage for every new token, over the keys it sees
 * (new token i of request r at absolute position p_r + i sees keys j <= p_r + i, the
 * bottom-right causal alignment of attn_extend_paged):
 *   S_j = sfQ[row][h] sfK[slot_j / 64][h_kv] (Q8 . K8_j),  m = max S_j,  l = sum exp(S_j - m),
 *   O[d] = sfV[h_kv][d] (sum_j E4M3(448 exp(S_j - m)) V8_j[d]) / (448 l) + v_mean[h_kv][d].
 * The dense Sage variant the pages measure at S = 10800 ("FlashInfer PrimTS, Sage
 * Attention ...", performance item 2).  Two passes over the key tiles of each query tile
 * (the row max first, then P8 and O) on the tcgen05 tensor cores in their 8-bit kinds:
 * Q8 . K8 on int8 (exact int32 dots), P8 . V8 on E4M3 with fp32 accumulation.
 *
 * params, d_ws    an EXTEND plan (attn_plan, mode PA_MODE_EXTEND) with page_size 64.
 * d_q8 int8 [max_q_tokens][Hq][D] (rows cu_seqlens_q[r] .. of request r), d_sf_q fp32
 *                 [max_q_tokens][Hq] (one scale per token and head).
 * Pools, sfK, sfV, v_mean and the table as for attn_decode_paged_sage; d_out bf16
 * [max_q_tokens][Hq][D].  q8, the pools and out 16-byte aligned.
 */
pa_status attn_extend_paged_sage(const pa_plan_params* params, const void* d_ws, size_t ws_bytes,
                                 const int8_t* d_q8, const float* d_sf_q, const int8_t* d_k8_pool,
                                 const uint8_t* d_v8_pool, const float* d_sf_k, const float* d_sf_v,
                                 const float* d_v_mean, int64_t num_slots, const int32_t* d_page_table,
                                 int64_t pt_pitch, uint16_t* d_out, pa_stream_t stream);

/*
 * attn_decode_paged_noalloc - attn_plan followed by attn_decode_paged in one
 * call, for callers that cannot allocate device memory (a host framework that
 * owns every device allocation and offers no allocator, a plugin that must not
 * touch its host process's memory pool, or a call site where an allocation
 * would synchronise the device or exceed a fixed memory budget).  The pages
 * have no counterpart to this entry point; it exists for such callers.
 *
 * Arguments are those of attn_plan (mode PA_MODE_DECODE, no cu_seqlens_q) and
 * attn_decode_paged, without the workspace: the plan, work list and split
 * partials live in a 16 MiB array inside the library, which every GPU that
 * loads the library holds until the process exits.  The call allocates and
 * frees nothing.  Plans whose pa_plan_workspace_size() exceeds 16 MiB are
 * rejected with PA_ERR_WORKSPACE (the Llama-3-8B decode shape, batch 64 x
 * Hq 32 on 148 SMs, needs about 6 MB).  The first call on a device looks up
 * the array's device address (once per device, with that device current); make
 * that first call before any stream capture.  All calls share the array and it
 * keeps the last call's contents: calls that overlap on the GPU (other streams
 * or host threads) race and must be ordered by the caller.  The device address
 * is kept for the life of the process: after cudaDeviceReset (or anything else
 * that destroys the device's primary context) this entry point must not be
 * called again in that process.  Device-side errors (an out-of-range page id, a
 * length beyond max_kv_len) are recorded in the array's header: read and clear
 * them with pa_noalloc_read_device_error.
 */
pa_status attn_decode_paged_noalloc(const pa_plan_params* params, const int32_t* d_seq_lens,
                                    const uint16_t* d_q, const uint16_t* d_k_pool,
                                    const uint16_t* d_v_pool, int64_t num_slots,
                                    const int32_t* d_page_table, int64_t pt_pitch, float sm_scale,
                                    uint16_t* d_out, float* d_lse_out, pa_stream_t stream);

/*
 * pa_noalloc_read_device_error - pa_read_device_error for attn_decode_paged_noalloc:
 * synchronise `stream`, read the device error word of the library's fixed
 * workspace array on the current device and clear it.  Returns PA_OK if clean,
 * PA_ERR_DEVICE_INDEX if the last calls met an out-of-range slot or page id or
 * length, PA_ERR_WORKSPACE if no no-allocation plan has been made on this device,
 * PA_ERR_CUDA on a CUDA error.  Allocates nothing.  (No counterpart on the pages.)
 */
pa_status pa_noalloc_read_device_error(pa_stream_t stream);

/*
 * attn_kv_store - write the K and V rows of new tokens into their pool slots: the cache
 * update that precedes attention in a forward pass ("Flash Attention Backend in SGLang:
 * Grundlagen und KV Cache optimal nutzen": the cache is updated within the forward
 * methods; the slot of each new token, out_cache_loc, comes from the caller's allocator).
 *
 *   k_pool[out_cache_loc[t]][h][:] = k_new[t][h][:],  the same for V, t < n_tokens.
 *
 * d_k_new, d_v_new   bf16 [n_tokens][Hkv][D], device, 16-byte aligned.
 * d_out_cache_loc    int32 [n_tokens], device: destination slot of each token.
 * d_k_pool, d_v_pool bf16 [num_slots][Hkv][D], device, 16-byte aligned.
 * d_ws               optional plan workspace: a slot outside [0, num_slots) is skipped and,
 *                    when d_ws is given, recorded in its error word (pa_read_device_error).
 * Two tokens with the same slot race (the last write wins, unspecified which).
 */
pa_status attn_kv_store(const uint16_t* d_k_new, const uint16_t* d_v_new, const int32_t* d_out_cache_loc,
                        int64_t n_tokens, int32_t hkv, int32_t head_dim, uint16_t* d_k_pool,
                        uint16_t* d_v_pool, int64_t num_slots, void* d_ws, pa_stream_t stream);

/*
 * attn_kv_store_sage - the same cache update for the 8-bit Sage pools, plus their K
 * scales:
 *   k8_pool[s][h][:] = k8_new[t][h][:],  v8_pool[s][h][:] = v8_new[t][h][:],
 *   sf_k[s / 64][h] = sf_k_new[t][h]  only when s % 64 == 0,
 * s = out_cache_loc[t].  The K scales are per 64-slot block ("FlashInfer PrimTS, Sage
 * Attention ...", README formula, sfK[blkK]); a block's scale is written by the token
 * whose slot opens the block, and later tokens of the block are expected to be quantised
 * (by the caller) with the scale already there.  The pages have no store step for 8-bit
 * pools; this is that reading.
 *
 * d_k8_new int8, d_v8_new E4M3 bytes, both [n_tokens][Hkv][D], device, 16-byte aligned.
 * d_sf_k_new  fp32 [n_tokens][Hkv] or NULL (the scales are left unchanged).
 * d_k8_pool, d_v8_pool [num_slots][Hkv][D], 16-byte aligned; d_sf_k fp32 [num_slots/64][Hkv]
 *             (required with d_sf_k_new; num_slots a multiple of 64 then).
 * d_ws, races and out-of-range slots as for attn_kv_store.
 */
pa_status attn_kv_store_sage(const int8_t* d_k8_new, const uint8_t* d_v8_new, const float* d_sf_k_new,
                             const int32_t* d_out_cache_loc, int64_t n_tokens, int32_t hkv, int32_t head_dim,
                             int8_t* d_k8_pool, uint8_t* d_v8_pool, float* d_sf_k, int64_t num_slots,
                             void* d_ws, pa_stream_t stream);

/*
 * attn_debug_gather - copy, for request r and KV head h_kv, the slot ids and
 * the K rows the kernels gather: d_slots_out int32 [L], d_rows_out bf16 [L][D]
 * for positions 0 .. L-1, L = min(d_seq_lens[r], max_len).  Out-of-range ids
 * are written as -1 with zero rows.  A test hook for checking the slot/page
 * indexing bit for bit; same table convention as the run calls.
 */
pa_status attn_debug_gather(const int32_t* d_seq_lens, int32_t r, int32_t h_kv, int32_t hkv,
                            int32_t head_dim, int32_t page_size, int32_t max_len,
                            const uint16_t* d_k_pool, int64_t num_slots,
                            const int32_t* d_page_table, int64_t pt_pitch,
                            int32_t* d_slots_out, uint16_t* d_rows_out, pa_stream_t stream);

/*
 * pa_read_device_error - synchronise `stream`, read the workspace's device
 * error word and clear it.  PA_OK if clean, PA_ERR_DEVICE_INDEX if a kernel
 * recorded an out-of-range id or length, PA_ERR_WORKSPACE if a run kernel
 * found a workspace built for another mode, PA_ERR_CUDA on a CUDA error.
 */
pa_status pa_read_device_error(void* d_ws, pa_stream_t stream);

/* Static, human-readable name of a status code. */
const char* pa_status_string(pa_status status);

/* Library version as major * 10000 + minor * 100 + patch. */
int32_t pa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDATTN_H */
