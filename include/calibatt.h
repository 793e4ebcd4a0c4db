/*
 * calibatt.h -- C ABI of the calibrated block-sparse attention library.
 *
 * The method is CalibAtt, "Accelerating Text-to-Video Generation with
 * Calibrated Sparse Attention" (arXiv 2603.05503, paper page): an offline
 * calibration pass finds block-level sparsity that is stable across inputs
 * (Abstract; Figure 5(a)), the patterns are compiled into per-(layer, head,
 * timestep) attention operations (Abstract), and at inference only the kept
 * blocks are computed while the others are skipped (Abstract; Figure 5(b)
 * top).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every tensor argument is caller-owned DEVICE memory unless marked
 *    "host".  The library allocates no device memory: scratch comes from the
 *    caller through (workspace, workspace_bytes), sized by the matching
 *    *_workspace_size query.
 *  - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is
 *    the legacy default stream).  The only calls that synchronize the stream
 *    are those that read results back to the host: calibatt_compile_size,
 *    calibatt_compile, calibatt_timestep_clusters, calibatt_skiplist_sizes
 *    and calibatt_blocklist_kept.
 *  - Every call returns a status: CALIBATT_OK (0) or a negative code below.
 *    On a non-zero return nothing was launched unless the code is
 *    CALIBATT_E_CUDA (a launch error).  calibatt_last_error() returns a
 *    thread-local, human-readable description of the last failure.
 *  - Errors found on the device (a corrupt block list, a bounded wait that
 *    ran out) are written, first error wins, to the optional int32 device
 *    word `dev_status` (0 = no error); the kernel then skips the affected
 *    work and exits cleanly.  Nothing in the library asserts, traps or
 *    aborts.
 *  - Tensor layouts are row-major and contiguous.  Attention tensors are
 *    [B, H, Np, d] with Np the padded sequence length (a multiple of the
 *    block size) and N <= Np the real length; padding rows must be present
 *    in memory (their values are ignored for keys and overwritten for
 *    outputs).
 */
#ifndef CALIBATT_H
#define CALIBATT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream handle (binary-compatible with cudaStream_t / CUstream). */
typedef struct CUstream_st* calibatt_stream_t;

/* ---- status codes ---------------------------------------------------- */
#define CALIBATT_OK              0
#define CALIBATT_E_INVALID      -1 /* bad argument (null, size, alignment, range) */
#define CALIBATT_E_UNSUPPORTED  -2 /* valid but not implemented (dtype/d/block)   */
#define CALIBATT_E_CUDA         -3 /* a CUDA runtime/driver call failed           */
#define CALIBATT_E_TIMEOUT      -4 /* a bounded device-side wait ran out          */
#define CALIBATT_E_CORRUPT      -5 /* block list failed its device-side checks    */
#define CALIBATT_E_WORKSPACE    -6 /* workspace missing or too small              */

/* ---- element types and selection modes ------------------------------- */
#define CALIBATT_BF16 0 /* bfloat16 inputs/outputs, tensor-core path           */
#define CALIBATT_FP32 1 /* float32 inputs/outputs, CUDA-core (FFMA) path       */

#define CALIBATT_SELECT_TOPK   0 /* keep ceil(frac * nkb) blocks (param = frac)  */
#define CALIBATT_SELECT_ENERGY 1 /* keep energy mass >= 1 - eps (param = eps)    */

#define CALIBATT_DEDUP_NONE 0 /* every non-empty row gets its own pattern       */
#define CALIBATT_DEDUP_HASH 1 /* translation-relative row-pattern dedup         */
#define CALIBATT_DEDUP_HASH_WEAK 2 /* same result, deliberately weak hash that
                                      collides often (exercises the exact
                                      collision path; for testing)             */

/*
 * Compiled kept-block lists (the mask dictionary in compiled form).
 *
 * Rows are (map, query block) pairs in map-major order, row r = map * nqb +
 * qb, where a map is one (layer, timestep, head) mask with map id
 * (layer * T + timestep) * H + head.  Row r keeps the key blocks
 *     row_base[r] + pat_off[pat_ptr[p] .. pat_ptr[p+1]),  p = row_pat[r],
 * ascending.  Pattern 0 is the empty pattern (a row with no kept block has
 * row_base 0 and row_pat 0).  Offsets within a pattern are ascending and
 * the first is 0.  Rows that are translates of one another share a pattern
 * (the within-frame row repetition of the paper page's Figure 4(b)).
 * The plain CSR (csr_row_ptr, csr_col) is optional (NULL to skip).
 *
 * All pointer members are device pointers owned by the caller.  Integer
 * members are host values.
 */
typedef struct calibatt_blocklist {
  int32_t n_maps, n_q_blocks, n_k_blocks, block_q, block_k;
  int32_t* row_base;    /* [n_maps * n_q_blocks]                          */
  int32_t* row_pat;     /* [n_maps * n_q_blocks]                          */
  int32_t* pat_ptr;     /* [n_pat + 1]                                    */
  int16_t* pat_off;     /* [nnz_pat]                                      */
  int64_t* csr_row_ptr; /* [n_maps * n_q_blocks + 1] or NULL              */
  int16_t* csr_col;     /* [nnz] or NULL                                  */
  int32_t n_pat, nnz_pat;
  int64_t nnz;
} calibatt_blocklist;

/* Thread-local text of the last error (never NULL). */
const char* calibatt_last_error(void);

/* Library version: major * 10000 + minor * 100 + patch. */
int calibatt_version(void);

/* Number of kernel launches the library has issued in this process. */
uint64_t calibatt_launch_count(void);

/* Limit (nanoseconds) of every bounded device-side wait; default 2e9.
 * Also read once from the environment variable CALIBATT_SPIN_LIMIT_NS.     */
void calibatt_set_spin_limit_ns(uint64_t ns);
uint64_t calibatt_get_spin_limit_ns(void);

/*
 * calibatt_sparse_attn_fwd -- block-sparse attention forward.
 *
 * Paper page, Abstract ("compute the selected input-dependent connections
 * densely, and skip the unselected ones") and Figure 5(b) top (load the block
 * mask, skip the unset blocks).  For batch b, head h and real query row
 * i < N of query block qb = i / block_q, with map = map_offset + h:
 *     J(i)  = { j < N : block j / block_k is kept in row (map, qb) of bl }
 *     O_i   = sum_{j in J(i)} exp(scale q_i.k_j - m_i) v_j / sum_{j in J(i)} exp(scale q_i.k_j - m_i)
 *     LSE_i = m_i + ln sum_{j in J(i)} exp(scale q_i.k_j - m_i),   m_i = max_j scale q_i.k_j
 * Rows i >= N and rows whose J(i) is empty get O_i = 0, LSE_i = -inf.
 *
 *  q, k, v  [B, H, Np, d] of `dtype` (16-byte aligned); o the same shape
 *           and type (written); lse [B, H, Np] float32 or NULL.
 *  scale    the softmax scale (normally the float32 of 1/sqrt(d)).
 *  bl       host pointer to a compiled block list with n_q_blocks =
 *           Np / block_q and n_k_blocks = Np / block_k (Np a multiple of
 *           both, Np - N below either); map_offset + H <= bl->n_maps.  The
 *           mask is shared by the batch.  Key blocks that do not divide the
 *           query padding use calibatt_sparse_attn_fwd_qk.
 *  dev_status optional device int32 (see conventions).
 * Supported: CALIBATT_BF16 with d in {64, 128}, block_q = 128 and block_k
 * in {64, 80, 96, 128, 144} (tcgen05 tensor cores, fp32 accumulation, P
 * rounded to bf16 for the PV product; paper page, Table S6 compares these
 * key-block sizes); CALIBATT_FP32 with d in {64, 128}, block_q and block_k
 * in {64, 128} (FFMA).  At most 2048 key blocks per row.  Anything else
 * returns CALIBATT_E_UNSUPPORTED.
 * Errors: CALIBATT_E_INVALID for a NULL or unaligned tensor, a non-positive
 * size, N > Np, a scale that is not finite and positive, a block list whose
 * grid does not match Np / block, padding of a whole block or more, or maps
 * beyond bl->n_maps; CALIBATT_E_UNSUPPORTED as above or for B * H * Np >=
 * 2^31; CALIBATT_E_CUDA for a launch failure.  On the device a corrupt row
 * of the block list writes CALIBATT_E_CORRUPT to dev_status (that row's
 * output becomes 0 / -inf) and a wait that runs out CALIBATT_E_TIMEOUT.
 */
int calibatt_sparse_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                             int B, int H, int N, int Np, int d, int dtype, float scale,
                             const calibatt_blocklist* bl, int map_offset,
                             int32_t* dev_status, calibatt_stream_t stream);

/*
 * calibatt_sparse_attn_fwd_streamed -- the forward above for inputs and
 * output in host memory.
 *
 * Computes exactly what calibatt_sparse_attn_fwd computes (same kernel, same
 * results bit for bit), one chunk of heads at a time: the chunk's Q, K, V are
 * copied host -> device on an internal copy stream, the forward of the chunk
 * runs on `stream`, and its O (and LSE) are copied device -> host on a second
 * copy stream, so the copies of one chunk overlap the compute of its
 * neighbours.
 *  q_host, k_host, v_host  [B, H, Np, d] of `dtype` in host memory (read);
 *                    page-locked memory is needed for the copies to overlap.
 *  o_host            [B, H, Np, d] host memory (written); lse_host [B, H, Np]
 *                    float32 host memory or NULL.
 *  q_dev, k_dev, v_dev, o_dev  device staging buffers of the same shape,
 *                    owned by the caller (16-byte aligned; overwritten);
 *                    lse_dev [B, H, Np] float32 device, non-NULL exactly when
 *                    lse_host is.
 *  heads_per_chunk   heads per chunk (>= 1; clamped to H); chunks never span
 *                    two batch entries.
 * The other arguments are those of calibatt_sparse_attn_fwd and are checked
 * before anything is enqueued.  The copy streams are ordered after the work
 * already on `stream`, and on return `stream` is ordered after every copy of
 * this call: synchronise `stream` before reading o_host.  The copy streams
 * and their events are created on first use (per device) and kept; calls
 * from several host threads are serialised while they enqueue.
 * Errors: CALIBATT_E_INVALID / E_UNSUPPORTED as calibatt_sparse_attn_fwd
 * (nothing enqueued); CALIBATT_E_CUDA if a copy or event call fails (work
 * enqueued before the failure stays enqueued).
 */
int calibatt_sparse_attn_fwd_streamed(const void* q_host, const void* k_host, const void* v_host, void* o_host,
                                      float* lse_host, void* q_dev, void* k_dev, void* v_dev, void* o_dev,
                                      float* lse_dev, int B, int H, int N, int Np, int d, int dtype, float scale,
                                      const calibatt_blocklist* bl, int map_offset, int heads_per_chunk,
                                      int32_t* dev_status, calibatt_stream_t stream);

/*
 * calibatt_sparse_attn_fwd_qk -- the forward with different query and key
 * lengths: Nq real query rows (padded to Npq) attend to Nk real keys (padded
 * to Npk).  Used by the spatial-repetition path (paper page, Figure 5(b)
 * bottom, Table S4), whose gathered anchor queries are fewer than the keys.
 *  q, o  [B, H, Npq, d];  k, v  [B, H, Npk, d];  lse [B, H, Npq] or NULL.
 *  bl    block list with block_q = 128, n_q_blocks = Npq / 128 and
 *        n_k_blocks = Npk / block_k; Npq - Nq < 128, Npk - Nk < block_k.
 * bf16 only (CALIBATT_E_UNSUPPORTED otherwise); other arguments, semantics and
 * errors as calibatt_sparse_attn_fwd.
 */
int calibatt_sparse_attn_fwd_qk(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                                int Nq, int Npq, int Nk, int Npk, int d, int dtype, float scale,
                                const calibatt_blocklist* bl, int map_offset, int32_t* dev_status,
                                calibatt_stream_t stream);

/*
 * calibatt_gather_rows -- dst[p, i, :] = src[p, idx[i], :] for p < n_planes,
 * i < rows_dst; an index outside [0, rows_src) writes a zero row.
 * The spatial-repetition path (paper page, Figure 4 and Table S4) gathers the
 * anchor query rows with it and broadcasts each anchor's output row to the
 * rows it stands for.
 *  src [n_planes, rows_src, row_bytes], dst [n_planes, rows_dst, row_bytes]
 *  (device, 16-byte aligned, row_bytes a multiple of 16); idx [rows_dst]
 *  int32 device.  Asynchronous.
 * Errors: CALIBATT_E_INVALID for a NULL pointer, a non-positive size, a
 * row_bytes that is not a multiple of 16 or an unaligned src / dst.
 */
int calibatt_gather_rows(const void* src, void* dst, const int32_t* idx, int n_planes, int rows_src, int rows_dst,
                         int row_bytes, calibatt_stream_t stream);

/*
 * calibatt_anchor_rows -- the anchor rows of the spatial-repetition path
 * (paper page, Figure 5(b) bottom: attention is computed for k anchor query
 * rows per frame and broadcast to the neighbouring rows; Table S4: k of the
 * 30 spatial rows at 480p).  Host arithmetic only (no device work).
 *  anchors  host int32 [k] (written): anchor i = floor((i + 1/2) rows / k),
 *           evenly spaced and centred, ascending;
 *  nearest  host int32 [rows] (written): the anchor row every spatial row takes
 *           its output from (the nearest anchor, the lower one on a tie).
 * Errors: CALIBATT_E_INVALID unless 1 <= k <= rows and both pointers are set.
 */
int calibatt_anchor_rows(int rows, int k, int32_t* anchors, int32_t* nearest);

/*
 * calibatt_anchor_plan_size -- the gathered query count of the
 * spatial-repetition path for a frames x rows x cols video: nq = frames k cols
 * anchor tokens, padded to npq (a multiple of 128).  Host arithmetic only.
 * Errors: CALIBATT_E_INVALID for a bad geometry or k outside [1, rows].
 */
int calibatt_anchor_plan_size(int frames, int rows, int cols, int k, int* nq, int* npq);

/*
 * calibatt_anchor_plan -- the two index lists of the spatial-repetition path
 * (paper page, Figure 4 and Figure 5(b) bottom), computed on the device:
 *  idx_q  device int32 [npq] (written): idx_q[i] = token of gathered query i
 *         (anchor tokens ordered by frame, anchor, column); -1 for i >= nq;
 *  idx_o  device int32 [Np] (written): idx_o[t] = gathered row whose output
 *         video token t takes (same frame and column, nearest anchor row);
 *         -1 for t >= frames rows cols.
 * Use: q_anchor = gather(q, idx_q); O_anchor = forward(q_anchor, k, v) with
 * calibatt_sparse_attn_fwd_qk; O = gather(O_anchor, idx_o)
 * (calibatt_gather_rows).  Asynchronous on `stream`.
 * Errors: as calibatt_anchor_plan_size; CALIBATT_E_INVALID if an index list
 * is NULL or Np is below the video token count.
 */
int calibatt_anchor_plan(int frames, int rows, int cols, int k, int Np, int32_t* idx_q, int32_t* idx_o,
                         calibatt_stream_t stream);

/*
 * calibatt_spatial_similarity -- the spatial-similarity score of every head's
 * attention map for one input (paper page, Figure 4: the attention pattern
 * repeats across the spatial rows of a frame; Figure 6(a) plots a map's
 * "spatial similarity"; Figure S13 flags heads whose score exceeds
 * tau = 0.87).  The pages do not define the score; this library reads it as
 * the mean, over the video query tokens (f, r, c) with r < rows - 1, of the
 * cosine similarity between the dense attention rows (softmax over all N real
 * keys) of tokens (f, r, c) and (f, r + 1, c), the two rows the anchor
 * broadcast (Figure 5(b) bottom) would give the same output.  Rows of P are
 * non-negative, so scores lie in [0, 1].
 *  q, k       [H, Np, d] bf16 device; tokens t < frames rows cols are the video
 *             (t = (f rows + r) cols + c), any further real tokens (< N, e.g.
 *             text) are keys only;
 *  score_out  [H] float32 device (written);
 *  workspace  device, >= calibatt_spatial_similarity_workspace_size bytes.
 * bf16, d in {64, 128}; N, Np as calibatt_block_energy; rows >= 2.
 * Deterministic (fixed-order reductions); asynchronous on `stream`.
 * Errors: CALIBATT_E_INVALID / E_UNSUPPORTED / E_WORKSPACE as the other calls
 * (nothing launched); device timeouts go to dev_status.
 */
int calibatt_spatial_similarity_workspace_size(int H, int Np, size_t* bytes);
int calibatt_spatial_similarity(const void* q, const void* k, int H, int N, int Np, int d, int dtype, int frames,
                                int rows, int cols, float scale, float* score_out, void* workspace,
                                size_t workspace_bytes, int32_t* dev_status, calibatt_stream_t stream);

/*
 * calibatt_repetition_flags -- the repetition dictionary (paper page, Figure
 * 5(a): heads that show spatial row repetition are stored in a dictionary;
 * Figure 6(b): the score varies little across calibration prompts; Figure
 * S13: tau = 0.87): per map, the mean score over the calibration inputs and
 * the flag mean >= tau.
 *  scores     [n_inputs, n_maps] float32 device (one calibatt_spatial_similarity
 *             per input, map id = (l T + t) H + h);
 *  mean_out   [n_maps] float32 device (written; may be NULL): the float32 sum
 *             in input order divided by n_inputs;
 *  flags_out  [n_maps] uint8 device (written): 1 where mean >= tau.
 * Asynchronous.  Errors: CALIBATT_E_INVALID for NULL pointers, bad sizes or a
 * non-finite tau.
 */
int calibatt_repetition_flags(const float* scores, int n_inputs, int n_maps, float tau, float* mean_out,
                              uint8_t* flags_out, calibatt_stream_t stream);



/*
 * calibatt_block_energy -- block energies of one calibration input.
 *
 * Paper page, Figure 2 (block-level post-softmax attention maps) and
 * Table S5 ("block energies"):
 *     E[h, qb, kb] = (1 / #rows(qb)) sum_{i in qb, i < N} sum_{j in kb, j < N} softmax_j(scale q_i.k_j)
 * with the softmax over ALL keys j < N (dense, unmasked).  Every row of E
 * sums to 1.  The key grid covers the real keys: nkb = ceil(N / block_k)
 * blocks, the last one partial when block_k does not divide N.
 *  q, k       [H, Np, d] of `dtype`, Np a multiple of block_q, Np - N < block_q;
 *  energy_out [H, Np/block_q, ceil(N/block_k)] float32 (written).
 *  workspace  >= calibatt_calibrate_workspace_size bytes (256-byte aligned).
 * Supported: CALIBATT_BF16 with d in {64,128}, block_q = 128 and block_k in
 * {64, 80, 96, 128, 144} (the key-block sizes of Table S6), at most 2 048
 * query blocks and 2 048 key blocks (tensor cores);
 * CALIBATT_FP32 with d in {64,128}, block_q and block_k in {64,128}, Np also
 * a multiple of block_k with Np - N < block_k (FFMA).
 * Errors: CALIBATT_E_INVALID (NULL, sizes, scale), CALIBATT_E_UNSUPPORTED
 * (shape outside the list), CALIBATT_E_WORKSPACE (workspace too small).
 * Asynchronous; dev_status (may be NULL) receives CALIBATT_E_TIMEOUT if a
 * bounded wait in the kernel expired.
 */
int calibatt_block_energy(const void* q, const void* k, int H, int N, int Np, int d, int dtype,
                          int block_q, int block_k, float scale, float* energy_out,
                          void* workspace, size_t workspace_bytes, int32_t* dev_status,
                          calibatt_stream_t stream);

/* Workspace bytes needed by calibatt_block_energy / calibatt_calibrate. */
int calibatt_calibrate_workspace_size(int H, int N, int Np, int d, int block_q, int block_k,
                                      size_t* bytes);

/*
 * calibatt_select_vote -- per-row selection of one input's energies, added
 * into the vote counts.
 *
 * Paper page, Figure 5(a) (threshold the top key blocks per query block) and
 * Figure 3(b) (how often each block is kept across calibration prompts).
 * Per row (h, qb), key blocks are ordered by (energy descending, index
 * ascending).  TOPK keeps the first k = min(nkb, max(1, ceil(frac * nkb)));
 * ENERGY keeps the shortest prefix whose float64 running sum reaches
 * (1 - eps) * (float64 sum of the row in index order), the crossing block
 * included.  Then votes[h,qb,kb] += kept and energy_sum[h,qb,kb] += E
 * (float32).
 *  energy      [H, nqb, nkb] float32 (read);  votes_inout int32, energy_sum_inout
 *              float32, both [H, nqb, nkb] (read-modify-write).
 * Errors: CALIBATT_E_INVALID for a NULL pointer, a non-positive size, an
 * unknown mode or a parameter out of range (frac in (0, 1], eps in [0, 1));
 * CALIBATT_E_UNSUPPORTED for nkb > 2048 or H * nqb >= 2^31.  Asynchronous on
 * `stream`; nothing is enqueued for a rejected call.
 */
int calibatt_select_vote(const float* energy, int H, int nqb, int nkb, int select_mode,
                         double select_param, int32_t* votes_inout, float* energy_sum_inout,
                         calibatt_stream_t stream);

/*
 * calibatt_finalize_mask -- agreement threshold (paper page, Figure 7, rho).
 * mask = votes >= min_votes.  A row left empty keeps exactly one key block:
 * the one with the most votes, then the largest energy_sum, then the
 * smallest index.  votes int32 and energy_sum float32 [H, nqb, nkb] (read);
 * mask_out [H, nqb, nkb] uint8 (0/1).
 * Errors: CALIBATT_E_INVALID for a NULL pointer, a non-positive size or
 * min_votes < 0; CALIBATT_E_UNSUPPORTED for H * nqb >= 2^31.  Asynchronous on
 * `stream`; nothing is enqueued for a rejected call.
 */
int calibatt_finalize_mask(const int32_t* votes, const float* energy_sum, int H, int nqb, int nkb,
                           int min_votes, uint8_t* mask_out, calibatt_stream_t stream);

/*
 * calibatt_calibrate -- the calibration pass over n_inputs inputs.
 *
 * For each input: calibatt_block_energy, then calibatt_select_vote into
 * votes_inout / energy_sum_inout (so repeated calls resume calibration:
 * the counts simply add up).  If mask_out != NULL, finishes with
 * calibatt_finalize_mask(min_votes).
 *  q_list, k_list  HOST arrays of n_inputs device pointers, each [H, Np, d].
 *  votes_inout, energy_sum_inout, mask_out  [H, Np/block_q, ceil(N/block_k)].
 * Shapes as calibatt_block_energy.
 * Errors: those of calibatt_block_energy (for every input), of
 * calibatt_select_vote and, when mask_out is set, of calibatt_finalize_mask;
 * CALIBATT_E_INVALID for n_inputs < 0 or NULL lists.  All arguments are
 * checked before the first launch, so a rejected call enqueues nothing.
 */
int calibatt_calibrate(const void* const* q_list, const void* const* k_list, int n_inputs,
                       int H, int N, int Np, int d, int dtype, int block_q, int block_k,
                       float scale, int select_mode, double select_param,
                       int32_t* votes_inout, float* energy_sum_inout, int min_votes,
                       uint8_t* mask_out, void* workspace, size_t workspace_bytes,
                       int32_t* dev_status, calibatt_stream_t stream);

/*
 * Compile masks [n_maps, nqb, nkb] (uint8, non-zero = kept) into a
 * calibatt_blocklist (paper page, Abstract: the patterns are compiled into
 * attention operations for each layer, head and timestep).  Patterns are
 * numbered in order of first occurrence over rows scanned in ascending
 * order; pattern 0 is the empty pattern.  nkb must be <= 32767.
 *
 * Two phases.  calibatt_compile_size computes the sizes (nnz = kept blocks,
 * n_pat = patterns incl. the empty one, nnz_pat = pattern-pool length) and
 * synchronizes the stream.  The caller then allocates the arrays, sets the
 * pointer members and the capacities n_pat / nnz_pat / nnz of `out`, and
 * calls calibatt_compile, which fills them, writes n_maps .. block_k, and
 * synchronizes; it fails with CALIBATT_E_INVALID if the capacities are
 * smaller than the sizes.  Workspace: calibatt_compile_workspace_size.
 * Errors: CALIBATT_E_INVALID for a NULL pointer, a non-positive size, an
 * unknown dedup mode or (compile) output capacities below the sizes;
 * CALIBATT_E_UNSUPPORTED for nkb > 32767, n_maps * nqb >= 2^31 or a pattern
 * pool beyond int32 indexing; CALIBATT_E_WORKSPACE for a missing or short
 * workspace; CALIBATT_E_CUDA if a launch or the read-back fails.
 */
int calibatt_compile_workspace_size(int n_maps, int nqb, int nkb, size_t* bytes);
int calibatt_compile_size(const uint8_t* masks, int n_maps, int nqb, int nkb, int dedup,
                          int64_t* nnz, int32_t* n_pat, int32_t* nnz_pat,
                          void* workspace, size_t workspace_bytes, calibatt_stream_t stream);
int calibatt_compile(const uint8_t* masks, int n_maps, int nqb, int nkb, int dedup,
                     int block_q, int block_k, calibatt_blocklist* out,
                     void* workspace, size_t workspace_bytes, calibatt_stream_t stream);

/*
 * calibatt_block_energy_noalloc -- calibatt_block_energy for callers that
 * cannot allocate device memory.
 *
 * The paper has no counterpart: this is a deployment variant.  Some callers
 * hold only their input and output buffers -- a plugin whose host engine
 * hands it no workspace, or a service that reserved the GPU's memory for its
 * own pool at start-up and allows no allocation afterwards -- so they cannot
 * supply the per-row scratch that calibatt_block_energy takes as workspace.
 * This entry point keeps that scratch in a fixed array inside the library's
 * device memory (16 MiB, held on every GPU that loads the library until the
 * process exits) and allocates nothing.  Same arguments, result and
 * supported shapes as calibatt_block_energy, minus the workspace.
 *
 *  - H * Np must be <= 4 194 304 (the array holds one float per query row);
 *    larger calls return CALIBATT_E_WORKSPACE and launch nothing.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture on the device.
 *  - Every call shares the one array.  Calls on one stream are ordered;
 *    calls that overlap on the GPU (other streams, other threads on the same
 *    device) race on the scratch and must not be issued.
 */
int calibatt_block_energy_noalloc(const void* q, const void* k, int H, int N, int Np, int d, int dtype,
                                  int block_q, int block_k, float scale, float* energy_out,
                                  int32_t* dev_status, calibatt_stream_t stream);

/*
 * calibatt_timestep_clusters -- groups the timesteps of every layer whose
 * calibrated masks are alike, so that they can share one mask.
 *
 * Paper page, Figure S11 (IoU of the skipped-block masks of two timesteps,
 * averaged over layers and heads; later, consecutive timesteps are alike) and
 * Table S3 (timestep sharing clusters masks with pair-wise IoU >= tau).
 * For layer l, the similarity of timesteps t1, t2 is the mean over heads h of
 *     |S(l,t1,h) & S(l,t2,h)| / |S(l,t1,h) | S(l,t2,h)|,  S = blocks with mask 0
 * (1 when both masks skip nothing).  Timesteps are grouped into runs of
 * consecutive steps, greedily in time order: step t joins the current run
 * when its similarity with every member is >= tau, otherwise it starts a new
 * run.  Runs are numbered globally in (layer, time) order.
 *  masks      [L, T, H, nqb, nkb] uint8 device (nonzero = kept; map order
 *             (l T + t) H + h).
 *  run_of     host int32 [L * T] (written): the run of every (l, t);
 *  n_runs     host int32 (written): the number of runs.
 *  workspace  device, >= calibatt_timestep_clusters_workspace_size bytes,
 *             256-byte aligned.
 * Synchronizes the stream (the grouping runs on the host from exact integer
 * pair counts computed on the device).  T <= 1024.
 * Errors: CALIBATT_E_INVALID for a NULL pointer, a non-positive size or a NaN
 * tau; CALIBATT_E_UNSUPPORTED for T > 1024 or L * T > 2^20;
 * CALIBATT_E_WORKSPACE for a short or unaligned workspace.
 */
int calibatt_timestep_clusters_workspace_size(int L, int T, int H, size_t* bytes);
int calibatt_timestep_clusters(const uint8_t* masks, int L, int T, int H, int nqb, int nkb, double tau,
                               int32_t* run_of, int32_t* n_runs, void* workspace, size_t workspace_bytes,
                               calibatt_stream_t stream);

/*
 * calibatt_share_masks -- one mask per run: the union of the kept blocks of
 * the run's members (nothing any member keeps is skipped).
 *  masks     [L, T, H, nqb, nkb] uint8 device;  run_of_dev device int32
 *            [L * T] as returned by calibatt_timestep_clusters;
 *  shared    [n_runs, H, nqb, nkb] uint8 device (written, 0/1).
 * The call (l, t) then uses map_offset = run_of[l T + t] * H of the shared
 * dictionary.  Asynchronous on `stream`.
 * Errors: as calibatt_timestep_clusters for the sizes; CALIBATT_E_INVALID for
 * n_runs outside [1, L * T]; CALIBATT_E_UNSUPPORTED for n_runs * H > 65535.
 * Run indices in run_of_dev outside [0, n_runs) select no run (harmless).
 */
int calibatt_share_masks(const uint8_t* masks, int L, int T, int H, int nqb, int nkb, const int32_t* run_of_dev,
                         int n_runs, uint8_t* shared, calibatt_stream_t stream);

/*
 * calibatt_interval_counts -- the number of intervals (maximal runs of
 * consecutive kept key blocks) of every row of a mask dictionary: the row
 * length of the paper page's interval skip lists (Figure S9, Figure S10).
 *  masks   [n_maps, nqb, nkb] uint8 device (nonzero = kept);
 *  counts  [n_maps * nqb] int32 device (written).  Asynchronous.
 * Errors: CALIBATT_E_INVALID for a NULL pointer or a non-positive size.
 */
int calibatt_interval_counts(const uint8_t* masks, int n_maps, int nqb, int nkb, int32_t* counts,
                             calibatt_stream_t stream);

/*
 * calibatt_merge_intervals -- merges outlier rows (paper page, Figure S10 (c)
 * and Table S3): every row of map i with more than width[i] intervals has
 * its smallest gaps (runs of skipped blocks between two kept blocks; ties to
 * the leftmost gap) filled until width[i] intervals remain.  Filled blocks
 * become kept (they are computed; the mask loses that much sparsity).
 *  masks   [n_maps, nqb, nkb] uint8 device, modified in place; nkb <= 2048.
 *  width   [n_maps] int32 device (values below 1 count as 1).
 *  filled  one uint64 on the device: the number of filled blocks is added.
 * Asynchronous.
 * Errors: CALIBATT_E_INVALID for a NULL pointer or a non-positive size;
 * CALIBATT_E_UNSUPPORTED for nkb > 2048.
 */
int calibatt_merge_intervals(uint8_t* masks, int n_maps, int nqb, int nkb, const int32_t* width,
                             unsigned long long* filled, calibatt_stream_t stream);

/*
 * calibatt_skiplist_sizes -- sizes of the paper page's padded per-layer
 * interval skip lists (Figure S10, Table S3) from the interval counts of a
 * mask dictionary (calibatt_interval_counts).  A layer is maps_per_layer
 * consecutive maps (all of its timesteps and heads); its array has one row per
 * (map, query block) and one slot per interval (an int32 pair, 8 bytes):
 *  full     ceil(nkb / 2) slots per row (the most a row can need);
 *  trimmed  the layer's largest count (layer_max);
 *  merged   for each percentile pcts[p] in (0, 100], the nearest-rank
 *           percentile of the layer's counts: the smallest count c such that
 *           at least ceil(pcts[p] / 100 * rows) counts are <= c
 *           (layer_width); rows above it are merged to it with
 *           calibatt_merge_intervals, which fills their smallest gaps.
 *  counts       device int32 [n_maps * nqb];
 *  layer_max    host int32 [n_layers] (written), n_layers = n_maps / maps_per_layer;
 *  layer_width  host int32 [n_pcts * n_layers] (written), percentile-major;
 *  map_width    device int32 [n_pcts * n_maps] (written) or NULL: each map's
 *               layer width per percentile, the width argument of
 *               calibatt_merge_intervals (map_width + p * n_maps);
 *  bytes        host int64 [2 + n_pcts] (written): full, trimmed, then merged
 *               for each percentile;
 *  workspace    device, >= calibatt_skiplist_sizes_workspace_size bytes.
 * Synchronizes `stream`.  nkb <= 16384, n_pcts <= 64.
 * Errors: CALIBATT_E_INVALID for bad sizes or percentiles, CALIBATT_E_WORKSPACE
 * for a short workspace, CALIBATT_E_CUDA if a copy fails.
 */
int calibatt_skiplist_sizes_workspace_size(int n_maps, int maps_per_layer, int n_pcts, size_t* bytes);
int calibatt_skiplist_sizes(const int32_t* counts, int n_maps, int nqb, int nkb, int maps_per_layer,
                            const double* pcts, int n_pcts, int32_t* layer_max, int32_t* layer_width,
                            int32_t* map_width, int64_t* bytes, void* workspace, size_t workspace_bytes,
                            calibatt_stream_t stream);

/*
 * calibatt_blocklist_bytes -- bytes of this library's compiled forms of a
 * mask dictionary, for comparison with the skip lists: the plain CSR (int64
 * row pointers, int16 columns) and the pattern pool (int32 base and pattern
 * id per row, int32 pattern pointers, int16 offsets); sizes from
 * calibatt_compile_size.  Host arithmetic only.
 * Errors: CALIBATT_E_INVALID for NULL outputs or sizes out of range.
 */
int calibatt_blocklist_bytes(int n_maps, int nqb, int64_t nnz, int32_t n_pat, int32_t nnz_pat, int64_t* csr_bytes,
                             int64_t* pool_bytes);

/*
 * calibatt_min_votes -- the integer agreement threshold of the vote (paper
 * page, Figure 3(b) and Figure 7: a block is kept when at least a fraction rho
 * of the calibration inputs keep it): min_votes = ceil(rho n_inputs), with
 * rho n_inputs rounded to 9 decimals first (so 0.3 * 10 gives 3), clamped to
 * [0, n_inputs].  Host arithmetic only.
 * Errors: CALIBATT_E_INVALID for a NULL output, n_inputs <= 0 or a rho that is
 * not finite.
 */
int calibatt_min_votes(double rho, int n_inputs, int32_t* min_votes);

/*
 * calibatt_topk_count -- key blocks kept per query-block row by the top-k
 * selection (paper page, Figure 5(a)): ceil(frac nkb) clamped to [1, nkb], the
 * count calibatt_select_vote uses.  Host arithmetic only; frac in (0, 1].
 * Errors: CALIBATT_E_INVALID for a NULL output, nkb <= 0 or frac outside (0, 1].
 */
int calibatt_topk_count(double frac, int nkb, int32_t* k);

/*
 * calibatt_blocklist_kept -- the number of kept blocks of maps [map_offset,
 * map_offset + n_maps) of a compiled block list (the sum of their rows'
 * pattern lengths), for per-call density and FLOP counts.  workspace: 8 bytes
 * of device memory (8-byte aligned).  Synchronizes `stream`.
 * Errors: CALIBATT_E_INVALID for a NULL pointer, maps outside the list or an
 * unaligned workspace; CALIBATT_E_WORKSPACE for a workspace under 8 bytes;
 * CALIBATT_E_CUDA if the launch or the read-back fails.
 */
int calibatt_blocklist_kept(const calibatt_blocklist* bl, int map_offset, int n_maps, int64_t* kept, void* workspace,
                            size_t workspace_bytes, calibatt_stream_t stream);

/*
 * calibatt_selftest_wait_timeout -- launches one block that waits, with the
 * bounded wait every kernel here uses, on a barrier that nothing completes.
 * After `limit_ns` it gives up and writes CALIBATT_E_TIMEOUT to dev_status.
 * Lets a caller check the timeout path without faulting or hanging a GPU.
 * Errors: CALIBATT_E_INVALID for a NULL dev_status or a limit outside
 * (0, 10 s].
 */
int calibatt_selftest_wait_timeout(uint64_t limit_ns, int32_t* dev_status,
                                   calibatt_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* CALIBATT_H */
