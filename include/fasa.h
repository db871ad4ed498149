/*
 * fasa.h -- C ABI of the FASA decode hot path on NVIDIA B200 (sm_100a).
 *
 * FASA ("FASA: Frequency-aware Sparse Attention", Wang et al.) predicts which
 * cached tokens matter for the current query from a few RoPE frequency chunks
 * (FCs), keeps the top-k of them, and runs exact softmax attention over only
 * those rows. Citations below name the page and section that define each step:
 *
 *   [abstract]  chatpaper.ai page "FASA: Frequency-aware Sparse Attention",
 *               English abstract.
 *   [tech §2]   gist.science page "FASA: Frequency-aware Sparse Attention",
 *               "Resumo Técnico" (technical summary), §2 "Metodologia e
 *               Insight Central": "A Descoberta" (FCs), the TIP bullets
 *               (offline calibration, online prediction), the FAC bullets,
 *               and "Variantes de Implementação" (FASA-M / FASA-C).
 *
 * Notation: B batch, Hq query heads, Hkv KV heads, G = Hq / Hkv query heads
 * per KV head (query head h belongs to KV head h / G), d = 128 head dim,
 * 64 FCs; FC i is the dim pair (i, i + 64) ("rotate-half" pairing) rotated at
 * theta_i = rope_base^(-2i/128). A cached token in slot t sits at absolute
 * position t. "dtype" is the cache dtype, used for keys, values, queries and
 * outputs alike.
 *
 * Conventions shared by every call:
 *  - All pointers are DEVICE pointers owned by the caller, 16-byte aligned,
 *    tensors dense and row-major as documented. The library allocates no
 *    memory; fasa_decode takes a caller-owned workspace.
 *  - Calls are asynchronous on `stream` (0 = legacy default stream) and do not
 *    synchronize, except fasa_device_status.
 *  - Arguments are validated on the host before anything is launched; a
 *    rejected call launches nothing and returns an error status. A CUDA launch
 *    failure returns FASA_ERR_CUDA. No call aborts, throws, or traps the GPU.
 *  - Problems only the device can see (an out-of-range token index given to
 *    fasa_sparse_attend, an out-of-range dominant-FC index, a bounded wait
 *    that gave up) are recorded in a sticky per-device status word, read by
 *    fasa_device_status. The offending element is skipped, never accessed.
 *  - Thread safety: calls may be made from several host threads; the only
 *    library state is the per-device status word and cached device attributes.
 *  - q_pos, where a call takes it, is the query's absolute position (>= 0) or
 *    FASA_Q_PREROTATED for queries the caller has rotated already.
 */
#ifndef FASA_H_
#define FASA_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FASA_ABI_VERSION 1
#define FASA_HEAD_DIM 128
#define FASA_NUM_FC 64
#define FASA_MAX_GROUP 16          /* largest G = Hq / Hkv */
#define FASA_MAX_LEN (1 << 19)     /* largest cached length a decode call accepts */
#define FASA_MAX_K (1 << 17)       /* largest kept-token budget */
#define FASA_CAL_MAX_WIN 8         /* calibration queries per calibration call */
/* A query position meaning "q is already rotated" (RoPE applied by the
 * caller): the library applies no rotation. Accepted wherever a call takes
 * q_pos (not by the calibration calls). Rotation at angle 0 is the identity,
 * so this equals rotating by position 0. */
#define FASA_Q_PREROTATED (-1)

typedef enum fasa_status {
  FASA_OK = 0,
  FASA_ERR_INVALID_ARG = 1,   /* null / misaligned pointer, bad size or range */
  FASA_ERR_UNSUPPORTED = 2,   /* head_dim != 128, G > 16, len > FASA_MAX_LEN, ... */
  FASA_ERR_CAPACITY = 3,      /* write or read beyond max_len */
  FASA_ERR_WORKSPACE = 4,     /* workspace missing or too small */
  FASA_ERR_CUDA = 5,          /* a CUDA runtime call or launch failed */
  FASA_ERR_TIMEOUT = 6,       /* device: a bounded wait gave up (status word) */
  FASA_ERR_BAD_INDEX = 7      /* device: an index outside its range was skipped */
} fasa_status;

typedef enum fasa_dtype { FASA_F32 = 0, FASA_BF16 = 1 } fasa_dtype;

/*
 * A KV cache of one attention layer, with its dominant-FC key sketch.
 *
 *  k, v    : [B][Hkv][max_len][128] dtype. Slot t of (b, g) holds the key
 *            rotated at position t (RoPE applied at append time) and the
 *            unrotated value.
 *  sketch  : [B][Hkv][max_len][sketch_stride] dtype. Row t of (b, g) holds,
 *            for j = 0 .. n_dom-1, element 2j = k[b][g][t][dom[g][j]] and
 *            element 2j+1 = k[b][g][t][dom[g][j] + 64] (the two dims of
 *            dominant FC j, copied from the stored rotated key); elements
 *            2*n_dom .. sketch_stride-1 are zero. It is what TIP reads, so a
 *            decode step streams 2*n_dom values per token instead of 256
 *            ([tech §2] FASA-C reads only a sparse subset of key state;
 *            FASA-M keeps the dominant key parts on the GPU apart from the
 *            rest).
 *  dom_idx : [Hkv][n_dom] int32, the dominant FCs I_dom of each KV head from
 *            offline calibration ([tech §2] TIP, first bullet): distinct,
 *            each in [0, 64). fasa_check_dom_idx validates a host copy.
 *  sketch_stride must equal fasa_sketch_stride(n_dom, dtype).
 */
typedef struct fasa_cache {
  int32_t batch;          /* B >= 1 */
  int32_t n_q_heads;      /* Hq, a multiple of Hkv */
  int32_t n_kv_heads;     /* Hkv >= 1 */
  int32_t head_dim;       /* must be 128 */
  int32_t n_dom;          /* 1 .. 64 */
  int32_t max_len;        /* capacity in tokens, 1 .. 2^30 */
  int32_t dtype;          /* fasa_dtype */
  int32_t sketch_stride;  /* elements per sketch row */
  double rope_base;       /* > 1 */
  void* k;
  void* v;
  void* sketch;
  const int32_t* dom_idx;
} fasa_cache;

/* ABI version (FASA_ABI_VERSION of the built library). */
int32_t fasa_abi_version(void);

/* Human-readable name of a status code (static string, never NULL). */
const char* fasa_status_string(int32_t status);

/* Description of the CUDA error behind the calling thread's most recent
 * FASA_ERR_CUDA (static string, never NULL; "no error" before any). */
const char* fasa_last_cuda_error(void);

/* Sketch row length in elements for n_dom dominant FCs: 2*n_dom rounded up
 * so that a row is a power-of-two number of 16-byte chunks (so a 16-byte load
 * never straddles two tokens). Returns -1 for n_dom outside 1..64 or an
 * unknown dtype. */
int32_t fasa_sketch_stride(int32_t n_dom, int32_t dtype);

/* Host-side check of a HOST copy of dom_idx ([Hkv][n_dom]): FASA_OK when
 * every row holds distinct values in [0, 64), else FASA_ERR_INVALID_ARG. */
fasa_status fasa_check_dom_idx(const int32_t* dom_idx_host, int32_t n_kv_heads, int32_t n_dom);

/*
 * FASA-M, the memory-optimised variant ([tech §2] "Variantes de
 * Implementação": the value cache and the non-dominant key parts are moved
 * to CPU memory, only what scoring needs stays on the GPU; [tech §4]
 * Eficiência/Compressão: 8x smaller KV cache on the GPU).
 *
 * A cache is FASA-M when its k and v point into pinned host memory that the
 * device can address, while sketch and dom_idx stay in device memory. Then
 * the GPU holds 2*n_dom of the 256 K and V values of a token (8x less at
 * n_dom = 16). The keys are kept whole on the host (their dominant dims are
 * also in the sketch), so the attention reads a kept row in one piece. Every
 * call works on such a cache unchanged:
 *  - fasa_append_kv writes K_rot and V through the host link and the sketch
 *    to device memory.
 *  - A decode streams the sketch from HBM, selects, and then reads only the
 *    k_eff kept K and V rows of each (b, g) across the host link, 2 * 128 *
 *    es bytes per kept token. The fused plan reads them with its split-K
 *    attention launch (many CTAs keep more requests on the link) also for
 *    budgets it would attend inside the fused kernel on a device-resident
 *    cache, so fasa_decode_launches counts 2 or 3 there.
 *  - fasa_dense_decode reads all of K and V across the link (correct, slow;
 *    bf16 caches only: FASA_ERR_UNSUPPORTED for an f32 FASA-M cache).
 *
 * fasa_host_kv_pointer returns in *device_ptr the address under which the
 * device reads the pinned host range starting at host_ptr, for use as
 * fasa_cache.k or .v. The range must lie in an allocation pinned with
 * cudaHostAlloc / cudaMallocHost (mapped; with unified addressing every such
 * allocation is) or registered with cudaHostRegister(cudaHostRegisterMapped).
 * Errors: NULL arguments or memory the device cannot address ->
 * FASA_ERR_INVALID_ARG (no CUDA error is left pending).
 */
fasa_status fasa_host_kv_pointer(void* host_ptr, void** device_ptr);

/*
 * Append n_new tokens at positions pos0 .. pos0+n_new-1 of every sequence.
 * [tech §2] "A Descoberta" (RoPE rotates each FC at its own frequency) and
 * FAC (positions are kept absolute): each key is rotated at its own position
 * once, here, and stored rotated.
 *
 *  k_new, v_new : [B][Hkv][n_new][128] dtype, pre-RoPE keys and values.
 *  Writes k, v and sketch rows pos0 .. pos0+n_new-1 of every (b, g).
 *  Arithmetic: cos/sin and the rotation in float64, rounded once to dtype
 *  (round to nearest even).
 *  Errors: FASA_ERR_CAPACITY when pos0 + n_new > max_len; n_new == 0 is a
 *  no-op returning FASA_OK.
 */
fasa_status fasa_append_kv(const fasa_cache* cache, const void* k_new, const void* v_new,
                           int32_t n_new, int32_t pos0, cudaStream_t stream);

/*
 * TIP online prediction ([tech §2] TIP, second bullet; [abstract]: the
 * dominant FCs are a computationally free proxy for token importance).
 * For every sequence b, KV head g and cached token t < len:
 *   scores[b][g][t] = sum over the G query heads h of g, and over the
 *   dominant FCs i of g, of  q'_h[i] k[t][i] + q'_h[i+64] k[t][i+64],
 * where q'_h is query h rotated at position q_pos.
 *
 *  q      : [B][Hq][128] dtype, pre-RoPE queries.
 *  scores : [B][Hkv][len] float32 (row stride len).
 *  Arithmetic: the query rotation and the group sum of each sketch column's
 *  coefficient c_j in float64, rounded once to float32; the score is then a
 *  float32 sum of products in a fixed order (the same in every plan of
 *  fasa_decode), with |error| < 13.01 * 2^-24 * sum_j |c_j| |sketch_j|.
 *  len may be 0 (nothing is written). Errors: FASA_ERR_CAPACITY if
 *  len > max_len.
 */
fasa_status fasa_score(const fasa_cache* cache, int32_t len, const void* q, int32_t q_pos,
                       float* scores, cudaStream_t stream);

/*
 * Critical-set selection T_t ([tech §2] FAC, first bullet): for each of
 * n_rows score rows, the indices of the k_eff = min(k, len) largest scores;
 * equal scores go to the lower index (-0.0 counts as +0.0); indices are
 * written in ascending order. Exact (radix select on order-preserving keys).
 *
 *  scores : [n_rows][len] float32, finite.
 *  idx    : [n_rows][k_eff] int32.
 *  Errors: k < 1, len < 1 or n_rows < 1 -> FASA_ERR_INVALID_ARG;
 *  len > FASA_MAX_LEN or k > FASA_MAX_K -> FASA_ERR_UNSUPPORTED.
 */
fasa_status fasa_select_topk(const float* scores, int32_t n_rows, int32_t len, int32_t k,
                             int32_t* idx, cudaStream_t stream);

/*
 * Focused attention ([tech §2] FAC, second and third bullets): full softmax
 * attention of each query head over only the given rows of its KV head,
 * each row at its original absolute position (keys were rotated at append):
 *   out[b][h] = sum_j softmax_j(q'_h . k[idx_j] / sqrt(128)) v[idx_j].
 *
 *  q    : [B][Hq][128] dtype, pre-RoPE (rotated here at q_pos).
 *  idx  : [B][Hkv][n_idx] int32, each in [0, len); duplicates count twice.
 *         An index outside [0, len) is skipped and recorded as
 *         FASA_ERR_BAD_INDEX in the device status word.
 *  out  : [B][Hq][128] dtype.
 *  Arithmetic: float32 logits and online softmax, output rounded to dtype.
 *  Errors: n_idx < 1 or len < 1 -> FASA_ERR_INVALID_ARG.
 */
fasa_status fasa_sparse_attend(const fasa_cache* cache, int32_t len, const void* q, int32_t q_pos,
                               const int32_t* idx, int32_t n_idx, void* out, cudaStream_t stream);

/* Workspace bytes fasa_decode needs for this cache at cached length len and
 * budget k (0 for invalid arguments). */
size_t fasa_decode_workspace_bytes(const fasa_cache* cache, int32_t len, int32_t k);

/*
 * One FASA decode step over a layer: TIP (fasa_score) -> T_t
 * (fasa_select_topk with k) -> FAC (fasa_sparse_attend), with results equal
 * to those three calls in sequence (the same float32 scores, hence the same
 * kept set). Two launch plans compute it:
 *
 *  FASA_DECODE_FUSED  (bf16 caches) each (batch, KV head) row is spread over
 *    about (SM count / rows) independent CTAs. Each scores its share of the
 *    sketch in registers, keeps its own top-k candidates and publishes them
 *    to the workspace; the row's last CTA to finish (an atomic ticket, no
 *    waiting) selects the exact top-k of the union and, for k_eff <= 256
 *    and G <= 8, attends those rows itself: one launch. Larger budgets add
 *    a split-K attention launch over the kept list (and, when a row's list
 *    spans several CTAs, a launch that merges their partial results).
 *  FASA_DECODE_STAGED  four launches chained with programmatic dependent
 *    launch: the score stream, which also builds a per-row histogram of the
 *    score keys and, in the row's last CTA, the row's threshold bin; a
 *    filter that marks the certainly-kept tokens and collects
 *    the tokens of the threshold bin; a per-row exact resolution of that bin
 *    that emits the kept indices in ascending order; and the focused
 *    attention (plus the split merge when a row's kept list spans several
 *    CTAs). Scores, histogram and index lists live in the workspace.
 *
 *  out     : [B][Hq][128] dtype.
 *  idx_out : nullable; [B][Hkv][min(k, len)] int32, the kept tokens in
 *            ascending order.
 *  workspace : caller-owned device memory of at least
 *            fasa_decode_workspace_bytes(cache, len, k) bytes, 256-byte aligned
 *            (required whichever plan runs). Zero it once after allocating it
 *            (e.g. cudaMemsetAsync): it starts with per-row semaphores,
 *            histograms, counters and tickets, at offsets that depend on
 *            B * Hkv only, which must be zero when a call starts and which
 *            every call leaves zero again; the rest is scratch. So one
 *            workspace sized for the largest len and k serves calls at any
 *            smaller len and k on the same cache. After a
 *            call that ended in an error (a CUDA error, FASA_ERR_TIMEOUT),
 *            zero it again. A semaphore found non-zero is reported as
 *            FASA_ERR_WORKSPACE in the device status word; no access then
 *            leaves the workspace.
 *  Ordering: the kernels of a plan follow one another with programmatic
 *  dependent launch, but every read of q, the cache and the workspace
 *  happens after all work issued earlier on the stream has completed (each
 *  plan's first kernel waits on the preceding grid before reading); only
 *  L2 prefetch hints and the kernels' own parameters may be read earlier.
 *  Calls that overlap on the GPU (different streams) must not share a
 *  workspace.
 *  Errors: as fasa_score, fasa_select_topk and fasa_sparse_attend;
 *  FASA_ERR_WORKSPACE if the workspace is missing or too small;
 *  FASA_ERR_UNSUPPORTED if fasa_set_decode_path forced FASA_DECODE_FUSED on a
 *  shape it cannot take.
 */
fasa_status fasa_decode(const fasa_cache* cache, int32_t len, const void* q, int32_t q_pos,
                        int32_t k, void* out, int32_t* idx_out, void* workspace,
                        size_t workspace_bytes, cudaStream_t stream);

/* Launch plan of fasa_decode (library code, no counterpart in the paper). */
#define FASA_DECODE_AUTO 0   /* chosen from the shape (default) */
#define FASA_DECODE_FUSED 1  /* row-split decode: one launch (k_eff <= 256, G <= 8), else 2-3 */
#define FASA_DECODE_STAGED 2 /* score, filter, finalize, attend (and the split merge): 4-5 launches */

/* Sets the plan every later fasa_decode call of this process uses (a
 * process-wide setting; FASA_ERR_INVALID_ARG for an unknown value). */
fasa_status fasa_set_decode_path(int32_t path);

/* The plan fasa_decode would run for this cache, len and k under the current
 * setting and on the current device: FASA_DECODE_FUSED or FASA_DECODE_STAGED,
 * or a negative fasa_status for invalid arguments. */
int32_t fasa_decode_path(const fasa_cache* cache, int32_t len, int32_t k);

/* Kernels of this library one fasa_decode call launches for this cache, len
 * and k under the current setting on the current device (the fused plan: 1,
 * or 2 when the budget needs the split-K attention; the staged plan: 4; the
 * split-K attention of a bf16 cache adds 1, the split merge, when a row's
 * kept list spans several CTAs), or a negative fasa_status for invalid
 * arguments. */
int32_t fasa_decode_launches(const fasa_cache* cache, int32_t len, int32_t k);

/*
 * Batches of sequences at different lengths, and per-KV-head budgets
 * ([tech §3] "Contribuições Principais", versatility: FASA works with
 * budgets allocated per layer and per head). The lengths live on the device
 * (a serving loop updates them without a host round trip); the host gives
 * upper bounds that size the launch and the workspace.
 *
 *  seq_len    : device [B] int32: sequence b holds cache slots 0 ..
 *               seq_len[b]-1 and its query sits at position seq_len[b]
 *               (or, with q_prerotated, is already rotated). Each value must
 *               lie in 1 .. max_seq_len; a value outside is clamped into that
 *               range and flagged FASA_ERR_BAD_INDEX in the status word.
 *  budget     : device [Hkv] int32, kept tokens for every sequence's KV head
 *               g, in 1 .. max_budget (clamped and flagged likewise), or
 *               NULL: max_budget for every head. A layer's call takes that
 *               layer's budgets, so budgets can differ per layer and per head.
 *  max_seq_len: host bound, 1 .. cache max_len and <= FASA_MAX_LEN.
 *  max_budget : host bound, 1 .. FASA_MAX_K.
 *  q_prerotated: 0: queries are pre-RoPE; 1: already rotated.
 */
typedef struct fasa_varlen {
  const int32_t* seq_len;
  const int32_t* budget;
  int32_t max_seq_len;
  int32_t max_budget;
  int32_t q_prerotated;
  int32_t reserved;
} fasa_varlen;

/* Workspace bytes fasa_decode_varlen needs (0 for invalid arguments). */
size_t fasa_decode_varlen_workspace_bytes(const fasa_cache* cache, const fasa_varlen* vl);

/*
 * fasa_decode over sequences of their own lengths with per-head budgets:
 * for every (b, g), the critical set of the k_eff = min(budget[g],
 * seq_len[b]) best-scoring tokens of slots 0 .. seq_len[b]-1 and the focused
 * attention of the group's query heads over it (results equal to fasa_decode
 * run on that sequence alone at its length and budget). Runs the fused plan
 * (bf16 caches): the kernels size their work from the device lengths.
 *
 *  q       : [B][Hq][128] dtype.
 *  out     : [B][Hq][128] dtype.
 *  idx_out : nullable; [B][Hkv][max_budget] int32: the kept tokens of (b, g)
 *            in ascending order, then -1 up to max_budget.
 *  workspace: as fasa_decode (zeroed once; at least
 *            fasa_decode_varlen_workspace_bytes bytes, 256-byte aligned).
 *  Errors: as fasa_decode; FASA_ERR_UNSUPPORTED for f32 caches.
 */
fasa_status fasa_decode_varlen(const fasa_cache* cache, const fasa_varlen* vl, const void* q, void* out,
                               int32_t* idx_out, void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Paged caches (serving realism, [tech §3] "Contribuições Principais",
 * Versatilidade: sequences of their own lengths sharing one pool). The
 * cache's k, v and sketch then point to page pools,
 *   k, v   : [n_pages][Hkv][block_size][128] dtype,
 *   sketch : [n_pages][Hkv][block_size][sketch_stride] dtype,
 * and slot t of sequence b, KV head g is row t % block_size of page
 * block_table[b][t / block_size], head g. fasa_cache.batch is the number of
 * sequences and fasa_cache.max_len must equal max_blocks * block_size (the
 * capacity of one sequence). Pages are owned and assigned by the caller.
 *
 *  block_table: device [B][max_blocks] int32. Every entry a call reaches
 *               (blocks 0 .. (slot)/block_size of the slots it reads or
 *               writes) must lie in 0 .. n_pages-1; an entry outside is
 *               flagged FASA_ERR_BAD_INDEX in the status word and its rows
 *               are skipped (not read, not written). The table is read on
 *               the device after the call's launch dependencies, so a kernel
 *               earlier in the stream may fill it.
 *  block_size : tokens per page, a power of two in 16 .. 65536.
 *  max_blocks : table row length (>= 1).
 *  n_pages    : pages in each pool; n_pages * Hkv * block_size < 2^31.
 */
typedef struct fasa_paged {
  const int32_t* block_table;
  int32_t block_size;
  int32_t max_blocks;
  int32_t n_pages;
  int32_t reserved;
} fasa_paged;

/*
 * fasa_append_kv into a paged (or, with pages NULL, contiguous) cache, each
 * sequence at its own position: the n_new tokens of sequence b go to slots
 * pos0[b] .. pos0[b]+n_new-1, rotated at those positions.
 *  pos0  : device [B] int32. A sequence whose range leaves 0 .. max_len-1 is
 *          skipped and flagged FASA_ERR_BAD_INDEX in the status word.
 *  k_new, v_new: [B][Hkv][n_new][128] dtype, device.
 *  Errors: as fasa_append_kv (host checks), invalid pages -> INVALID_ARG.
 */
fasa_status fasa_append_kv_paged(const fasa_cache* cache, const fasa_paged* pages, const void* k_new,
                                 const void* v_new, int32_t n_new, const int32_t* pos0, cudaStream_t stream);

/* Workspace bytes fasa_decode_paged needs (0 for invalid arguments). */
size_t fasa_decode_paged_workspace_bytes(const fasa_cache* cache, const fasa_paged* pages, const fasa_varlen* vl);

/*
 * fasa_decode_varlen over a paged cache: the same results as
 * fasa_decode_varlen on a contiguous cache holding the same slots (bf16
 * caches; kept indices are logical slots). Errors: as fasa_decode_varlen;
 * invalid pages -> FASA_ERR_INVALID_ARG.
 */
fasa_status fasa_decode_paged(const fasa_cache* cache, const fasa_paged* pages, const fasa_varlen* vl,
                              const void* q, void* out, int32_t* idx_out, void* workspace,
                              size_t workspace_bytes, cudaStream_t stream);

/*
 * Multi-query decode: n_q query tokens per sequence in one step (draft
 * tokens to verify, or several rows served together). Reading of the pages
 * for more than one query ([tech §2] TIP's group sum, FAC): the n_q * G
 * query rows of KV head g share one critical set, the k_eff best tokens by
 * s_t = sum_j sum_{h in g} sum_{i in D_g} P_i(q'_{j,h}, k'_t); each row then
 * attends over the kept slots that are not after its own position. Query
 * token j sits at position q_pos0 + j: with q_pos0 >= len (the usual case)
 * every kept slot is visible; with draft tokens already appended at
 * q_pos0 .. q_pos0 + n_q - 1 the rows see only what precedes them. A row
 * left with no visible kept slot is zero. With q_pos0 = FASA_Q_PREROTATED
 * the queries are used as given and nothing is masked.
 *
 * The attention runs on the tensor cores (tcgen05, accumulators in tensor
 * memory): Q K^T and P V over tiles of 128 kept rows, each bf16 operand
 * that is not stored in the cache (the scaled rotated queries, the
 * probabilities) split into two bf16 terms, float32 accumulation.
 *
 *  q       : [B][n_q][Hq][128] bf16.
 *  out     : [B][n_q][Hq][128] bf16.
 *  idx_out : nullable; [B][Hkv][k_eff] int32, ascending.
 *  n_q     : 1 .. 16, with n_q * G <= 64.
 *  workspace: zeroed once before first use, at least
 *            fasa_decode_multi_workspace_bytes(cache, len, n_q, k) bytes,
 *            256-byte aligned; every call leaves it ready for the next.
 *  Errors: as fasa_decode; n_q out of range or f32 caches ->
 *  FASA_ERR_UNSUPPORTED (n_q < 1 -> FASA_ERR_INVALID_ARG).
 */
size_t fasa_decode_multi_workspace_bytes(const fasa_cache* cache, int32_t len, int32_t n_q, int32_t k);
fasa_status fasa_decode_multi(const fasa_cache* cache, int32_t len, const void* q, int32_t q_pos0, int32_t n_q,
                              int32_t k, void* out, int32_t* idx_out, void* workspace, size_t workspace_bytes,
                              cudaStream_t stream);

/* Size of the library's own device scratch used by
 * fasa_decode_static_scratch: 64 MiB, held by every GPU that loads the
 * library until the process exits. */
#define FASA_STATIC_SCRATCH_BYTES ((size_t)64 << 20)

/*
 * fasa_decode for callers that cannot allocate device memory. (The paper has
 * no counterpart; this is a deployment convenience.) Some callers have no
 * way to obtain a workspace: a plugin running inside a host framework that
 * owns the whole device memory pool and hands its extensions no scratch, or
 * a latency-critical path that must not call cudaMalloc (it may synchronize
 * the device) and keeps no allocator of its own. This entry point computes
 * exactly what fasa_decode computes, but its scratch is a fixed array inside
 * the library (FASA_STATIC_SCRATCH_BYTES per device) instead of a caller
 * workspace. It allocates nothing. The caller still passes all inputs and
 * outputs.
 *
 *  - The first call on a device looks up that device's copy of the array
 *    (with that device current); make that first call before any stream
 *    capture. Later calls reuse the cached address.
 *  - Every call on a device shares the one array and leaves its last
 *    contents behind; calls whose kernels overlap on the GPU (different
 *    streams, or different host threads) race on it and give wrong results.
 *    Serialize them, e.g. on one stream.
 *  - Each call clears the array's per-row semaphores (a cudaMemsetAsync of
 *    12 * B * Hkv bytes on `stream`) before its kernels, so a call that
 *    ended in an error does not affect the next one.
 *  - Rejects a call needing more than FASA_STATIC_SCRATCH_BYTES of scratch
 *    (fasa_decode_workspace_bytes(cache, len, k)) with FASA_ERR_WORKSPACE,
 *    before launching anything.
 *  Other arguments and errors: as fasa_decode.
 */
fasa_status fasa_decode_static_scratch(const fasa_cache* cache, int32_t len, const void* q, int32_t q_pos,
                                       int32_t k, void* out, int32_t* idx_out, cudaStream_t stream);

/* Workspace bytes fasa_dense_decode needs for this cache and len (0 for
 * invalid arguments). */
size_t fasa_dense_workspace_bytes(const fasa_cache* cache, int32_t len);

/*
 * Dense full-KV decode, the comparison path: the same attention as
 * fasa_sparse_attend over all len cached rows (the upper bound in
 * [tech §4] "Resultados Experimentais", full KV "FKV"). bf16 caches run the
 * decode's split-K attention over every row (a one-wave grid of splits,
 * merged by a second launch; tensor-core products for groups of up to 8
 * query heads); f32 caches a cluster kernel.
 *
 *  workspace : at least fasa_dense_workspace_bytes(cache, len) bytes,
 *            256-byte aligned, zeroed once after allocation: its first
 *            4 * B * Hkv bytes are per-row counters that must be zero when a
 *            call starts and that every call leaves zero; the rest is scratch.
 *  Errors: as fasa_sparse_attend; FASA_ERR_WORKSPACE for a missing or short
 *  workspace.
 */
fasa_status fasa_dense_decode(const fasa_cache* cache, int32_t len, const void* q, int32_t q_pos,
                              void* out, void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Synchronizes the current device, then returns FASA_OK or the first
 * device-side problem recorded since the status was last cleared
 * (FASA_ERR_BAD_INDEX, FASA_ERR_TIMEOUT); clears it when clear != 0.
 * Returns FASA_ERR_CUDA if the synchronization itself fails.
 */
fasa_status fasa_device_status(int32_t clear);

/*
 * Offline calibration of the dominant FCs ([tech §2] TIP, first bullet: once,
 * before decoding, each head's I_dom is found from the "Contextual Agreement"
 * between the attention scores of a single FC and of the full head over a
 * small calibration set). The pages give no formula for the agreement; these
 * calls measure it as the overlap of the token sets the two scores select
 * at the decode budget, exactly as the decode selects them.
 *
 * Calibration query w of sequence b sits at position q_pos0 + w and attends
 * to the len cached rows of the cache (its keys, not its sketch). For KV
 * head g, with qs = the group's G rotated queries added head by head:
 *   plane i < 64 : P_i(t)  = qs[i] k[t][i] + qs[i+64] k[t][i+64]
 *   plane 64     : full(t) = P_0(t) + P_1(t) + ... + P_63(t)   (FC order)
 * each product and sum one float64 operation, the result rounded once to
 * float32. Then, with K_eff = min(budget, len) and Top_K the selection of
 * fasa_select_topk (ties to the lower index):
 *   counts[g][i] = sum over b and w of |Top_K(plane i) ∩ Top_K(plane 64)|
 *   dom_idx[g]   = the n_dom FCs with the largest counts, ties to the lower
 *                  FC index, in that order (a valid cache dom_idx row).
 */

/* Workspace bytes fasa_calibrate needs (0 for invalid arguments). */
size_t fasa_calibrate_workspace_bytes(const fasa_cache* cache, int32_t len, int32_t n_win, int32_t budget);

/*
 * The 65 score planes of every calibration query.
 *  q_win  : [B][n_win][Hq][128] dtype, pre-RoPE calibration queries.
 *  planes : [B][Hkv][n_win][65][len] float32 (row stride len).
 *  Errors: n_win outside 1..FASA_CAL_MAX_WIN, len < 1, q_pos0 < 0 or
 *  q_pos0 + n_win > 2^31 - 1 -> FASA_ERR_INVALID_ARG; len > max_len ->
 *  FASA_ERR_CAPACITY.
 */
fasa_status fasa_calibrate_scores(const fasa_cache* cache, int32_t len, const void* q_win, int32_t q_pos0,
                                  int32_t n_win, float* planes, cudaStream_t stream);

/*
 * Agreement counts from score planes laid out as fasa_calibrate_scores
 * writes them ([n_rows][n_win][65][len], n_rows = B * Hkv, row r belonging
 * to KV head r % n_kv_heads).
 *  counts    : [n_kv_heads][64] uint32, overwritten.
 *  workspace : at least n_rows * n_win * 65 * min(budget, len) * 4 bytes
 *              (the selections), 4-byte aligned.
 *  Errors: n_rows not a positive multiple of n_kv_heads, budget < 1,
 *  n_win outside 1..FASA_CAL_MAX_WIN or len < 1 -> FASA_ERR_INVALID_ARG;
 *  len > FASA_MAX_LEN or budget > FASA_MAX_K -> FASA_ERR_UNSUPPORTED;
 *  a short workspace -> FASA_ERR_WORKSPACE.
 */
fasa_status fasa_calibrate_counts(const float* planes, int32_t n_rows, int32_t n_kv_heads, int32_t n_win,
                                  int32_t len, int32_t budget, uint32_t* counts, void* workspace,
                                  size_t workspace_bytes, cudaStream_t stream);

/*
 * I_dom from counts: dom_idx [n_kv_heads][n_dom] int32 (device).
 *  Errors: n_kv_heads < 1 or n_dom outside 1..64 -> FASA_ERR_INVALID_ARG.
 */
fasa_status fasa_calibrate_dominant(const uint32_t* counts, int32_t n_kv_heads, int32_t n_dom, int32_t* dom_idx,
                                    cudaStream_t stream);

/*
 * The whole calibration: fasa_calibrate_scores into the workspace, then
 * fasa_calibrate_counts and fasa_calibrate_dominant. counts and dom_idx as
 * above; workspace of fasa_calibrate_workspace_bytes, 256-byte aligned.
 */
fasa_status fasa_calibrate(const fasa_cache* cache, int32_t len, const void* q_win, int32_t q_pos0, int32_t n_win,
                           int32_t budget, int32_t n_dom, uint32_t* counts, int32_t* dom_idx, void* workspace,
                           size_t workspace_bytes, cudaStream_t stream);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* FASA_H_ */
