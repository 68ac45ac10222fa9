/*
 * tria.h -- C ABI of the block-sparse mixed-precision causal attention library
 * (TriAttention-style), built for NVIDIA B200 (sm_100a).
 *
 * What is computed. Attention is cut into tiles of T query tokens x T key
 * tokens. Each tile of query block i and key block j (j <= i) gets one of three
 * actions -- skip, compute with 4-bit codes, compute with 8-bit codes -- from its
 * distance d = i - j to the diagonal and a per-head pair of boundaries
 * (hi, keep): 8-bit if d < hi, 4-bit if hi <= d < keep, skipped if d >= keep.
 * Key block 0 and the diagonal block are always computed with 8-bit codes.
 * (rit.work TriAttention page, section "Какие связи можно не считать, а какие
 * нельзя удалять", paragraphs three to five; the half-open bands and the
 * per-query-head pair are readings of that text.) All kept tiles of a query row
 * are reduced into one normalised softmax result, and the prepared K/V go to a
 * compressed KV cache that decode reads (section "Как калибровка распределяет
 * вычисления между головами", last paragraph).
 *
 * Codec (a reading; the page names only 4 and 8 bits): per token and per plane,
 * s = max|x| / 127 (int8) or max|x| / 7 (int4) in fp32 with IEEE division,
 * code = rint(x / s) with ties to even, clamped to [-127,127] / [-7,7]; an
 * all-zero row has scale 0 and codes 0. The tile's plane applies to Q, K and V.
 * Scores are (integer code dot product) * s_q * s_k / sqrt(D); softmax in fp32;
 * P.V in bf16 with fp32 accumulation. GQA maps query head h to KV head
 * h / (Hq / Hkv) (llmis.ru chapter 3.5, section 4).
 *
 * Conventions for every call:
 *  - Pointers named "device" are CUDA device pointers; "host" are host memory.
 *  - bf16 tensors are contiguous, row-major, [B, H, tokens, D] ("BHSD").
 *  - Device pointers must be 16-byte aligned; the workspace 256-byte aligned.
 *  - All memory is owned by the caller; the library allocates nothing.
 *  - Calls are asynchronous on `stream` (a cudaStream_t passed as void*,
 *    NULL = legacy default stream) and return a tria_status at once. Argument
 *    errors are found on the host before any launch and leave memory untouched.
 *  - Supported: D in {64, 128}, T in {64, 128}, Hq % Hkv == 0, Hq/Hkv <= 16,
 *    Hq <= 256, B <= 1024, device compute capability 10.0 (sm_100a).
 *  - Kernels never trap. A pipeline wait that runs past its limit, or an index
 *    that fails its check, sets an error word in the workspace and the kernel
 *    returns; tria_workspace_status() reports it.
 */
#ifndef TRIA_H_
#define TRIA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TRIA_OK = 0,
  TRIA_ERR_INVALID_ARG = 1,   /* bad shape, pointer, alignment or policy */
  TRIA_ERR_UNSUPPORTED = 2,   /* D, T, head ratio or GPU not supported */
  TRIA_ERR_CUDA = 3,          /* a CUDA runtime/driver call failed */
  TRIA_ERR_TIMEOUT = 4,       /* a device-side pipeline wait ran past its limit */
  TRIA_ERR_BOUNDS = 5,        /* a device-side index check failed */
  TRIA_ERR_WORKSPACE = 6      /* workspace missing or smaller than required */
} tria_status;

/* Compressed KV cache: the "prepared K and V" of the method, one row per token.
 * For X in {k, v}, in the contiguous layout (block_table == NULL):
 *   x8        int8  [B, Hkv, capacity, D]      8-bit codes
 *   x4        uint8 [B, Hkv, capacity, D/2]    4-bit codes, two per byte:
 *                                              element 2m in the low nibble,
 *                                              element 2m+1 in the high nibble,
 *                                              4-bit two's complement
 *   x8_scale  fp32  [B, Hkv, capacity]         per-token scale of the 8-bit plane
 *   x4_scale  fp32  [B, Hkv, capacity]         per-token scale of the 4-bit plane
 * In the paged layout (block_table != NULL) the planes are a pool of num_pages
 * pages of T tokens of every KV head -- x8 [num_pages, Hkv, T, D], x4
 * [num_pages, Hkv, T, D/2], scales [num_pages, Hkv, T] -- and logical block j
 * (tokens [jT, jT + T)) of sequence b lives in page block_table[b * max_blocks
 * + j]; capacity = max_blocks * T tokens per sequence. block_table is a device
 * int32 array the caller owns and may change between calls (pages handed out
 * as a sequence grows). Pages written by one call must not be shared by two
 * sequences.
 * status is a device int, the cache's error word: a page id outside
 * [0, num_pages) met by any kernel sets TRIA_ERR_BOUNDS there and that access is
 * skipped (reads go to page 0 instead); tria_cache_status reads and clears it.
 * All pointers are device pointers, the planes 16-byte aligned; capacity is a
 * multiple of T. The struct itself is host memory, read during the call only.
 * tria_cache_init / tria_paged_cache_init fill it. */
typedef struct {
  int8_t* k8;
  uint8_t* k4;
  float* k8_scale;
  float* k4_scale;
  int8_t* v8;
  uint8_t* v4;
  float* v8_scale;
  float* v4_scale;
  int B, Hkv, D, T, capacity;
  const int32_t* block_table;   /* NULL: contiguous; else device int32 [B, max_blocks] */
  int max_blocks, num_pages;    /* paged layout only */
  int* status;                  /* device error word */
} tria_kv_cache;

/* Shape of a prefill: B sequences of S tokens, Hq query heads, Hkv KV heads. */
typedef struct {
  int B, Hq, Hkv, S, D, T;
} tria_dims;

/* Human-readable name of a status code (static string). */
const char* tria_status_string(int status);

/* Bytes needed to hold every plane and the status word of a contiguous cache
 * carved by tria_cache_init. */
size_t tria_cache_bytes(int B, int Hkv, int D, int T, int capacity);

/* Fill `cache` with plane pointers carved from one caller buffer `base`
 * (device, 256-byte aligned, at least tria_cache_bytes(...) bytes), contiguous
 * layout. Writes no device memory: the caller zeroes the buffer (or calls
 * tria_cache_status once) before the status word is read. Returns
 * TRIA_ERR_INVALID_ARG on a bad shape or alignment. */
int tria_cache_init(tria_kv_cache* cache, void* base, size_t bytes,
                    int B, int Hkv, int D, int T, int capacity);

/* Paged compressed cache (the "special KV-cache layout" the rit.work TriAttention
 * page, section "Когда TriAttention меняет планы инфраструктуры", paragraph four,
 * says a deployment must support; pages of T tokens named by a block table, as
 * paged KV caches do). Bytes of a pool of num_pages pages plus the status word. */
size_t tria_paged_cache_bytes(int num_pages, int Hkv, int D, int T);

/* Fill `cache` for a paged pool carved from `base` (device, 256-byte aligned,
 * at least tria_paged_cache_bytes(...) bytes) serving B sequences through
 * `block_table` (device int32 [B, max_blocks], caller-owned, read by every call
 * that uses the cache). Writes no device memory. Returns TRIA_ERR_INVALID_ARG
 * on a bad shape, alignment or NULL table. */
int tria_paged_cache_init(tria_kv_cache* cache, void* base, size_t bytes, int B, int Hkv, int D, int T,
                          int num_pages, const int32_t* block_table, int max_blocks);

/* Synchronise `stream`, return the cache's status word (TRIA_OK or
 * TRIA_ERR_BOUNDS after a page id out of range) and clear it. */
int tria_cache_status(const tria_kv_cache* cache, void* stream);

/* Codec over arbitrary rows (used for Q and by the tests).
 * Passage: rit.work TriAttention page, section "Какие связи можно не считать, а
 * какие нельзя удалять", paragraph three (blocks computed at 8 or at 4 bits);
 * the per-token symmetric rule above is a reading of it.
 * X: device bf16 [rows, D]. Outputs (device): c8 int8 [rows, D], s8 fp32
 * [rows], c4 uint8 [rows, D/2] packed as in the cache, s4 fp32 [rows].
 * Any of c4/s4 may be NULL to skip that plane. Bit-exact with the codec rule
 * above. */
int tria_quantize_rows(const void* X, int64_t rows, int D, int8_t* c8, float* s8,
                       uint8_t* c4, float* s4, void* stream);

/* Write the prepared K/V of S tokens into cache positions [start, start+S).
 * Passage: rit.work TriAttention page, section "Как калибровка распределяет
 * вычисления между головами", last paragraph -- the prepared keys and values go
 * into a compressed KV cache that step-by-step generation reads; the 8-bit and
 * 4-bit planes are the two precisions of section "Какие связи можно не считать, а
 * какие нельзя удалять", paragraph three. Both planes of every token are written,
 * because the plane a tile uses depends on the query block that reads it.
 * K, V: device bf16 [B, Hkv, S, D] (B, Hkv, D as in the cache).
 * Requires 0 <= start, start + S <= capacity, S >= 1. Any start is allowed, so
 * this also appends decode tokens one at a time (S = 1). Errors: INVALID_ARG on
 * a bad range or pointer, UNSUPPORTED off sm_100a; nothing is written then. */
int tria_quantize_kv(const void* K, const void* V, int S, int start,
                     const tria_kv_cache* cache, void* stream);

/* Tile counts of one head over nb x nb blocks (host-only helper):
 * out[0] = int8 tiles, out[1] = int4 tiles, out[2] = skipped causal tiles. */
int tria_count_tiles(int nb, int hi, int keep, int64_t* out);

/* The loads the fused prefill makes for one query head (host-only helper; the
 * kernel's producers follow the same plan). The tile action is the one of the
 * rit.work TriAttention page, section on which links may be skipped and which
 * must be kept, as tria_count_tiles counts it. Query tiles are 128 rows: one
 * query block at T = 128, two at T = 64; they are listed in ascending order and
 * each tile's loads in the order the kernel issues them. A load is 128 keys:
 * four int32 per load, (i0, j0, j1, plane): the tile's first query block, the key
 * blocks (j1 = j0 at T = 128; at T = 64 j1 is a second block of the same plane, or
 * -1 when j0 goes alone) and the plane, 8 or 4.
 * nb >= 0 blocks, T in {64, 128}, 0 <= hi <= keep. `plan` (host memory, may be
 * NULL) receives min(count, capacity) loads; *count receives the total.
 * Returns TRIA_ERR_INVALID_ARG on a bad argument or a NULL `count`, and
 * TRIA_ERR_BOUNDS if a tile's walked load count differs from the closed-form count
 * the kernel's producer uses (a self-check; it does not happen). */
int tria_prefill_load_plan(int nb, int T, int hi, int keep, int32_t* plan, int64_t capacity, int64_t* count);

/* Workspace bytes tria_prefill needs for `dims` (0 if dims are invalid). */
size_t tria_prefill_workspace_bytes(const tria_dims* dims);

/* Fused block-sparse mixed-precision causal prefill.
 * Passage: rit.work TriAttention page, section "Какие связи можно не считать, а
 * какие нельзя удалять", paragraphs three to five (per tile: skip, 4 bits or
 * 8 bits, from the distance to the diagonal and the head's two boundaries; key
 * block 0 and the diagonal always at 8 bits), and section "Как калибровка
 * распределяет вычисления между головами", last paragraph (one fused kernel
 * takes the kept blocks grouped by precision and reduces them into one
 * normalised result).
 * Q: device bf16 [B, Hq, S, D]; cache: holds K/V tokens [0, S) (written by
 * tria_quantize_kv); hi, keep: HOST int32 arrays of length Hq with
 * 0 <= hi <= keep (keep may exceed the block count). S % T == 0,
 * S <= capacity. O: device bf16 [B, Hq, S, D]; LSE: device fp32 [B, Hq, S],
 * natural log-sum-exp of the row's kept scaled scores. workspace: device,
 * 256-byte aligned, >= tria_prefill_workspace_bytes(dims). */
int tria_prefill(const void* Q, const tria_kv_cache* cache, const tria_dims* dims,
                 const int32_t* hi, const int32_t* keep, void* O, float* LSE,
                 void* workspace, size_t workspace_bytes, void* stream);

/* GQA-shared prefill (llmis.ru chapter 3.5, section 4: the query heads of a group
 * read the same K and V). When Hq / Hkv is even and every pair of query heads
 * (2k, 2k + 1) of the call has the same (hi, keep), the fused kernel serves both
 * heads of a pair from one CTA, so each kept K/V block is brought on chip once for
 * the two. Results are those of the per-head kernel. Enabled by default; this
 * sets the process-wide choice (enable = 0: always per head) and returns the
 * previous one. Host-only. */
int tria_prefill_gqa(int enable);

/* Prefill of a prompt held in host memory: the cache write of tokens [0, S) of K and
 * V (as tria_quantize_kv) and the fused prefill of Q (as tria_prefill, the same
 * computation: rit.work TriAttention page, section "Как калибровка распределяет
 * вычисления между головами", last paragraph), with the copies in and out overlapped
 * with the kernels. The work is split by (batch, KV head) group: group g's K, V and
 * its Hq/Hkv query heads' Q are copied in on copy_in_stream while group g - 1's
 * kernels run on `stream` and group g - 2's O and LSE are copied out on
 * copy_out_stream, through the slots of `staging`. When Hq/Hkv is a multiple of 4
 * the last group goes as two units of half its query heads (the first also writes
 * the group's cache rows), which halves the work left after the last copy in.
 *   hQ, hK, hV    host bf16, [B,Hq,S,D] and [B,Hkv,S,D]; page-locked memory lets the
 *                 copies overlap (pageable memory works, serialised by the runtime).
 *   hO, hLSE      host bf16 [B,Hq,S,D] and fp32 [B,Hq,S], written by the call.
 *   cache         contiguous cache (no block table) with B, Hkv, D, T of dims and
 *                 capacity >= S; its rows [0, S) of every group are written.
 *   hi, keep      host int32 [Hq], as tria_prefill.
 *   staging       device, 256-byte aligned, >= tria_prefill_host_staging_bytes(dims)
 *                 (two slots); a buffer of k slots' bytes, k <= 4, lets the copies in
 *                 run k - 1 groups ahead of the kernels.
 *   workspace     device, 256-byte aligned, >= tria_prefill_host_workspace_bytes(dims)
 *                 (the prefill workspace of one group); its status word is read with
 *                 tria_workspace_status.
 *   streams       three distinct streams. The call returns once everything is queued;
 *                 `stream` completes after the last copy out, so synchronising it (or
 *                 an event recorded on it after the call) makes hO and hLSE readable.
 * Returns TRIA_ERR_UNSUPPORTED for a paged cache, TRIA_ERR_INVALID_ARG for a
 * missing pointer, equal streams, a small buffer or dims that disagree with the
 * cache; the per-group calls' own checks and status codes otherwise. */
size_t tria_prefill_host_staging_bytes(const tria_dims* dims);
size_t tria_prefill_host_workspace_bytes(const tria_dims* dims);
int tria_prefill_host(const void* hQ, const void* hK, const void* hV, const tria_kv_cache* cache,
                      const tria_dims* dims, const int32_t* hi, const int32_t* keep,
                      void* hO, float* hLSE, void* staging, size_t staging_bytes,
                      void* workspace, size_t workspace_bytes, void* stream,
                      void* copy_in_stream, void* copy_out_stream);

/* The two halves of tria_prefill, for callers that time or schedule them apart.
 * tria_prefill_prepare: Q codec (both planes) and the operand tiles built from
 * the cache (4-bit K expanded to one code per byte, V dequantised to bf16 and
 * transposed per block) into `workspace`; reads Q and the cache only.
 * tria_prefill_attend: the fused block-sparse kernel over what prepare left in
 * the same workspace, for the same cache and dims; writes O and LSE.
 * prepare followed by attend on one stream equals tria_prefill. Arguments,
 * layouts and errors are those of tria_prefill. */
int tria_prefill_prepare(const void* Q, const tria_kv_cache* cache, const tria_dims* dims, void* workspace,
                         size_t workspace_bytes, void* stream);
int tria_prefill_attend(const tria_kv_cache* cache, const tria_dims* dims, const int32_t* hi,
                        const int32_t* keep, void* O, float* LSE, void* workspace, size_t workspace_bytes,
                        void* stream);

/* The work plan tria_decode launches with (host-only helper; the decode kernel's
 * producer maps each work item to a group and a run of its kept blocks from it). The
 * kept blocks are the union over a group's query heads of the blocks the tile action
 * keeps at the query position kv_len[b] - 1 (rit.work TriAttention page, section on
 * which links may be skipped and which must be kept). Per group g = b * Hkv + kvh:
 * nkept[g] kept blocks, split into ceil(nkept[g] / bps) items of at most bps blocks
 * (*blocks_per_split), its first item and partial slot split_start[g]
 * (split_start[B * Hkv] = *n_items). The kernel hands out every group's splits but
 * the first (the blocks nearest the diagonal, bps each) first, then the groups' first
 * splits (block 0 and the far band) in the order first_order lists the groups.
 * num_sms: the SMs the launch would use (the plan asks for about six items per SM).
 * Arguments as tria_decode (kv_len, hi, keep host int32); split_start has B * Hkv + 1
 * entries, first_order and nkept B * Hkv. Returns TRIA_ERR_INVALID_ARG or
 * TRIA_ERR_UNSUPPORTED as tria_decode would, TRIA_OK otherwise. */
int tria_decode_plan(int B, int Hq, int Hkv, int T, int capacity, const int32_t* kv_len, const int32_t* hi,
                     const int32_t* keep, int num_sms, int32_t* split_start, int32_t* first_order, int32_t* nkept,
                     int32_t* blocks_per_split, int32_t* n_items);

/* Workspace bytes tria_decode needs (0 if the arguments are invalid). */
size_t tria_decode_workspace_bytes(int B, int Hq, int Hkv, int D, int T, int capacity);

/* Split-KV decode of one new token per sequence over the compressed cache.
 * Passage: rit.work TriAttention page, section "Как калибровка распределяет
 * вычисления между головами", last paragraph (the chosen boundaries are used in
 * both stages; generation reads the prepared K/V from the compressed cache and so
 * reads less data), with decode bound by memory traffic (llmis.ru chapter 3.5,
 * section 2). The new token is one row of the prefill problem.
 * q: device bf16 [B, Hq, D]; kv_len: HOST int32 [B], 1 <= kv_len[b] <=
 * capacity: the token sits at position kv_len[b]-1 and is already in the
 * cache, so its block is the diagonal block. hi, keep: HOST int32 [Hq].
 * O: device bf16 [B, Hq, D]; LSE: device fp32 [B, Hq]. Only the kept blocks
 * of the planes some head of a KV group needs are read; partial results of
 * the splits are merged by log-sum-exp. */
int tria_decode(const void* q, const tria_kv_cache* cache, const int32_t* kv_len, int Hq,
                const int32_t* hi, const int32_t* keep, void* O, float* LSE,
                void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of the fixed device scratch array used by tria_decode_static. */
#define TRIA_DECODE_STATIC_SCRATCH_BYTES (40u << 20)

/* Split-KV decode without a caller workspace and without allocating.
 * No counterpart in the paper: this is a deployment convenience for callers
 * that cannot allocate device memory -- for example a plugin inside a host
 * application whose device memory is fully budgeted in advance, or a
 * latency-critical loop that must not call cudaMalloc, which may synchronise
 * the device. Arguments and results are those of tria_decode minus the
 * workspace. The scratch is one fixed __device__ array of
 * TRIA_DECODE_STATIC_SCRATCH_BYTES (40 MiB) inside this library, held by every
 * GPU that loads it until the process exits. Problems whose decode workspace
 * (tria_decode_workspace_bytes) is larger are rejected with
 * TRIA_ERR_WORKSPACE before anything runs. The first call on each device looks
 * up the array's device address (cudaGetSymbolAddress) with that device
 * current; make that first call before any stream capture. All calls on a
 * device share the array: each call clears what must start at zero, and calls
 * whose GPU work overlaps (unordered streams) race on it. The address is looked
 * up per CUDA context, so a context the caller created and made current gets its
 * own copy of the array. A device-side pipeline error (a wait past its limit)
 * makes that call's O and LSE NaN and lands in the array's error word, which
 * tria_decode_static_status reads. */
int tria_decode_static(const void* q, const tria_kv_cache* cache, const int32_t* kv_len, int Hq,
                       const int32_t* hi, const int32_t* keep, void* O, float* LSE, void* stream);

/* Synchronise `stream` and return the device-side error word of the fixed
 * scratch array that tria_decode_static uses in the current context (TRIA_OK,
 * TRIA_ERR_TIMEOUT or TRIA_ERR_BOUNDS); every tria_decode_static call clears it.
 * No counterpart in the paper. Allocates nothing. */
int tria_decode_static_status(void* stream);

/* ---- Calibration of the per-head boundaries and the global allocator ----
 * Passage: rit.work TriAttention page, section "Как калибровка распределяет
 * вычисления между головами", paragraphs one to three: candidate boundary pairs
 * are tried for every head; a candidate's error is measured after the output
 * projection and normalised by the energy of the layer's output; each candidate
 * has a cost counting whole processed blocks (query-key product, normalisation
 * of the weights, aggregation of the values); a global allocator adds work where
 * it lowers the error most. Readings: the reference output keeps every block at
 * 8 bits; error of head h = sum over its rows of ||(O_c - O_ref) W_O[h]||^2, with
 * W_O[h] the D rows of W_O that head h feeds; energy of head h = sum over rows of
 * ||O_ref W_O[h]||^2 (cross terms between heads dropped in both); a kept tile
 * costs 4 T^2 D + 4 T^2 at 8 bits and 2 T^2 D + 4 T^2 at 4 bits. */

/* Cost of each candidate (cand_hi[c], cand_keep[c]) for one head over nb x nb
 * causal blocks of T tokens, head dim D: host-only. cost: host int64 [C]. */
int tria_calibration_costs(int nb, int T, int D, const int32_t* cand_hi, const int32_t* cand_keep, int C,
                           int64_t* cost);

/* Workspace bytes tria_calibrate needs (0 if the arguments are invalid). */
size_t tria_calibrate_workspace_bytes(const tria_dims* dims, int d_model);

/* Errors of C candidate boundary pairs, applied to every head at once, on one
 * layer's calibration sample. Q: device bf16 [B, Hq, S, D]; cache: holds that
 * sample's K/V (tokens [0, S)); W_O: device bf16 [Hq * D, d_model], row-major
 * (row h * D + k is what output element k of head h multiplies). cand_hi,
 * cand_keep: HOST int32 [C]. Writes HOST err [C, Hq] (the unnormalised errors
 * E[c][h]) and energy [Hq]; the normalised error is E / sum(energy). Runs the
 * fused prefill once for the reference and once per candidate, then waits for
 * the stream (the results are host memory). Returns a device-side error word of
 * the prefill as tria_workspace_status does, else TRIA_OK. */
int tria_calibrate(const void* Q, const tria_kv_cache* cache, const tria_dims* dims, const void* W_O, int d_model,
                   const int32_t* cand_hi, const int32_t* cand_keep, int C, double* err, double* energy,
                   void* workspace, size_t workspace_bytes, void* stream);

/* Greedy global allocation (host-only). err: host double [C, H], cost: host
 * int64 [C, H]; every head starts at its cheapest candidate (then the lower
 * error, then the first); then, while the total cost stays within `budget`, the
 * single move of one head to a costlier candidate with a lower error that has the
 * largest error decrease per unit of added cost is taken (the first in
 * head-then-candidate order on equal ratios). choice: host int32 [H]. */
int tria_allocate(const double* err, const int64_t* cost, int C, int H, int64_t budget, int32_t* choice);

/* Synchronise `stream` and return the device-side error word of `workspace`
 * (TRIA_OK, TRIA_ERR_TIMEOUT or TRIA_ERR_BOUNDS); the word is cleared by
 * every tria_prefill / tria_decode call that uses this workspace. After a
 * decode whose wait ran past its limit, that call's O and LSE are NaN. */
int tria_workspace_status(const void* workspace, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* TRIA_H_ */
