/*
 * csa.h - C ABI of libcsa: the compressed sparse attention (CSA) layer of
 * DeepSeek-V4 and its dense heavily compressed (HCA) variant, on NVIDIA B200
 * (sm_100a).
 *
 * Sources for the operations (pages on DeepSeek-V4):
 *   [EL]  "Evidence Ledger" (mastering-deepseek-v4-architecture), sections
 *         "CSA" (Eqs 9-19), "HCA" (Eqs 20-26) and "Shared attention details"
 *         (Sec 2.3.3, Eq 27, Sec 2.3.4).
 *   [SY]  "DeepSeek-V4" study (shuhuayu.github.io), "03 / Two resolutions of
 *         history" (pooling formula, index-score formula, configuration
 *         table) and "06 / What grows with context" (entry payloads).
 *   [CA]  "DeepSeek-V4: What Remains After Compressing History?", Sec 1
 *         (shared normalisation with the sink), Sec 2 (ledger example),
 *         Sec 3 (causality boundary).
 *
 * Conventions shared by every entry point
 *   - Every tensor pointer is a DEVICE pointer owned by the caller; the
 *     library keeps no pointer after the call returns. Tensors are dense and
 *     row-major with the shapes given below; "[a,b,c]" lists dimensions from
 *     outermost to innermost. Base pointers must be 16-byte aligned.
 *   - Work is enqueued on `stream`; no call synchronises the stream except
 *     csa_sync_status(). Calls on different streams may run concurrently.
 *   - The library allocates no device memory. Kernels that need scratch take
 *     a caller-provided `workspace` whose size a *_workspace_size() query
 *     returns; passing less returns CSA_ERR_INVALID_ARG.
 *   - Arguments are checked on the host before any launch; a bad argument
 *     returns CSA_ERR_INVALID_ARG (or CSA_ERR_UNSUPPORTED for a legal but
 *     unimplemented shape/dtype) and launches nothing. A launch failure
 *     returns CSA_ERR_CUDA. Bounded device-side waits that give up record
 *     CSA_ERR_TIMEOUT in a device error word that csa_sync_status() reports.
 *   - Outputs are overwritten. Inputs are never written, except the
 *     caller-owned decode state and caches of csa_compress_decode().
 *   - Positions p are 0-based token indices of the sequence.
 *
 * Readings of the pages fixed by this ABI (each one is a parameter where it
 * is cheap):
 *   - visibility: a query at position p sees compressed entries
 *     s < n_vis(p) = floor((p + vis_offset) / m), clipped to the entries that
 *     exist; vis_offset = 1 reads the ledger's strict causality s < floor(t/m)
 *     with t 1-based, the same count as the source rule (p+1)//m that [CA]
 *     Sec 3 reports; vis_offset = 0 is the literal 0-based reading.
 *   - block 0 of CSA has no preceding block: its b-series candidates are
 *     absent from the softmax.
 *   - bias rows 0..m-1 weight the preceding-block (b-series) candidates in
 *     token order, rows m..2m-1 the own-block (a-series) candidates.
 *   - RMSNorm: x / sqrt(mean(x^2) + eps) * gain, over the full width.
 *   - RoPE on the last rope_dims dims, interleaved pairs (2i, 2i+1),
 *     theta_i = rope_base^(-2i/rope_dims); entry i sits at position i*m.
 *   - softmax scale 1/sqrt(c); the sink adds exp(z'_h) to the denominator
 *     and carries no value.
 */
#ifndef CSA_H_
#define CSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* csa_stream_t; /* a cudaStream_t; NULL = legacy default stream */

typedef enum {
  CSA_OK = 0,
  CSA_ERR_INVALID_ARG = 1,
  CSA_ERR_UNSUPPORTED = 2,
  CSA_ERR_CUDA = 3,
  CSA_ERR_TIMEOUT = 4,
  CSA_ERR_TOO_LARGE = 5 /* the call needs more scratch than the fixed buffer
                           of csa_index_topk_noalloc() holds */
} csa_status;

typedef enum {
  CSA_F32 = 0,
  CSA_BF16 = 1,
  /* Mixed compressed-entry storage for c = 512, rope_dims = 64 ([EL] Sec
   * 2.3.4; [SY] 06): dims 0..447 as FP8 E4M3 codes scaled by one FP32 factor
   * per row, dims 448..511 (the RoPE dims) as BF16. Row layout, 592-byte
   * stride: bytes [0,448) E4M3 codes, [448,576) 64 x BF16, [576,580) FP32
   * scale, [580,592) zero padding. value[i] = e4m3(code[i]) * scale for
   * i < 448. Writers use scale = max|x[0:448]| / 448 and
   * code = RNE-satfinite(x / scale), both divisions in IEEE FP32; a row whose
   * first 448 values are all zero gets scale 0 and zero codes. */
  CSA_FP8_MIXED = 2
} csa_dtype;

#define CSA_MIXED_ROW_BYTES 592
#define CSA_MAX_TOPK 2048

typedef struct {
  int m;            /* tokens per compressed entry: 4 (CSA) or 128 (HCA) */
  int overlap;      /* 1: CSA, 2m candidates per entry; 0: HCA, m candidates */
  int c;            /* entry width = attention head width; multiple of 16, <= 1024 */
  int rope_dims;    /* RoPE on the last rope_dims dims; even, <= c */
  double rope_base; /* RoPE base, 10000 */
  float eps;        /* RMSNorm epsilon, 1e-6 */
  int vis_offset;   /* 1: n_vis(p) = floor((p+1)/m) (default); 0: floor(p/m) */
  int n_win;        /* sliding-window length, 128 */
  int win_ring;     /* window rows: 0 = row j holds position j (prefill);
                       1 = ring buffer, row (j mod n_win) holds position j */
} csa_geom;

/* Human-readable name of a status code (static string). */
const char* csa_status_string(csa_status s);

/* Library version string (static). */
const char* csa_version(void);

/* Number of CUDA kernels this library has launched in the process so far
 * (all devices, all streams). Lets a caller count the library's work. */
uint64_t csa_kernel_launches(void);

/* Synchronises `stream`, then reads and clears the device error word that
 * bounded device-side waits set. Returns CSA_ERR_TIMEOUT if a wait gave up
 * since the last call, CSA_ERR_CUDA on a CUDA error, else CSA_OK. */
csa_status csa_sync_status(csa_stream_t stream);

/* ---------------------------------------------------------------------
 * csa_rmsnorm_rope - prepare rows for core attention.
 * [EL] "Shared attention details": RMSNorm on compressed KV entries just
 * before core attention; partial RoPE on the last 64 dims.
 * y_r = RoPE_{pos_r}(RMSNorm(x_r) * gain) for each of `rows` rows of width
 * g->c. pos_r = pos[r] if `pos` is non-NULL (device int64 [rows]), else
 * pos0 + r * pos_step.
 *   x    [rows, c] in_dtype (F32 or BF16)
 *   gain [c] FP32, NULL = all ones
 *   out  output rows of width c, out_dtype (F32, BF16), or mixed rows of
 *        CSA_MIXED_ROW_BYTES when out_dtype = CSA_FP8_MIXED (c = 512,
 *        rope_dims = 64 only). Row r is written to output row out_row[r]
 *        when `out_row` (device int64 [rows]) is non-NULL - e.g. slot
 *        b*n_win + (p mod n_win) of a decode window ring - else to row r.
 * --------------------------------------------------------------------- */
csa_status csa_rmsnorm_rope(const csa_geom* g, csa_dtype in_dtype, csa_dtype out_dtype,
                            const void* x, int64_t rows, const int64_t* pos, int64_t pos0,
                            int64_t pos_step, const float* gain, void* out,
                            const int64_t* out_row, csa_stream_t stream);

/* ---------------------------------------------------------------------
 * csa_quantize_mixed - store rows of width 512 in the CSA_FP8_MIXED layout
 * with no normalisation or rotation ([EL] Sec 2.3.4 mixed KV storage).
 *   x   [rows, 512] in_dtype (F32 or BF16);  out [rows] mixed rows.
 * --------------------------------------------------------------------- */
csa_status csa_quantize_mixed(csa_dtype in_dtype, const void* x, int64_t rows, void* out,
                              csa_stream_t stream);

/* ---------------------------------------------------------------------
 * csa_compress - prefill KV compressor for one sequence of T tokens.
 * [EL] "CSA" Eqs 9-12 and "HCA" Eqs 20-26; [SY] 03 pooling formula.
 * CSA (g->overlap = 1):
 *   C^a = H W_aKV, C^b = H W_bKV, Z^a = H W_aZ, Z^b = H W_bZ        ([T, c])
 *   entry i, channel ch: softmax over the 2m candidates
 *     r = 0..m-1   : (C^b, Z^b) of token (i-1)m + r, bias row r   (absent if i = 0)
 *     r = m..2m-1  : (C^a, Z^a) of token im + r - m, bias row r
 *   of (Z + bias)[r, ch], weighting C[r, ch]; then RMSNorm over c (gain)
 *   and RoPE at position i*m.
 * HCA (g->overlap = 0): one series (W_aKV, W_aZ), m candidates per entry
 *   (tokens im..im+m-1, bias rows 0..m-1); W_bKV, W_bZ must be NULL.
 *   H     [T, d] dtype (F32 or BF16)
 *   W_*   [d, c] dtype
 *   bias  [(1+overlap)*m, c] FP32
 *   gain  [c] FP32, NULL = ones
 *   E_out [floor(T/m), c] out_dtype (F32, BF16 or CSA_FP8_MIXED rows)
 * Tokens after the last complete block are not pooled.
 * workspace: csa_compress_workspace_size() bytes for the same dtype.
 * --------------------------------------------------------------------- */
size_t csa_compress_workspace_size(const csa_geom* g, csa_dtype dtype, int64_t T, int d);
csa_status csa_compress(const csa_geom* g, csa_dtype dtype, const void* H, int64_t T, int d,
                        const void* W_aKV, const void* W_bKV, const void* W_aZ,
                        const void* W_bZ, const float* bias, const float* gain,
                        csa_dtype out_dtype, void* E_out, void* workspace, size_t ws_bytes,
                        csa_stream_t stream);

/* ---------------------------------------------------------------------
 * csa_compress_decode - decode-time compressor: one new token per sequence.
 * Same equations as csa_compress, evaluated incrementally ([EL]
 * "Infrastructure", Sec 3.5.1: fixed-size state cache holding the tokens of
 * the not yet complete block; CSA also keeps the previous block's b-series,
 * [CA] Sec 2).
 *   h        [B, d] dtype: hidden state of the token at position pos[b]
 *   pos      [B] int64 device
 *   state    [B, csa_compress_decode_state_floats(g)] FP32, caller-owned,
 *            persistent across steps; zero it before a sequence starts.
 *   E_cache  [B, ldE, c] out_dtype (row stride CSA_MIXED_ROW_BYTES for mixed)
 * For every b, the projections of h[b] are stored into state; when
 * (pos[b]+1) % m == 0 the block i = pos[b]/m is complete and entry i is
 * pooled, normalised, rotated and written to E_cache[b, i] (i < ldE is the
 * caller's responsibility; entries i >= ldE are skipped).
 * Tokens must arrive in position order per sequence.
 * workspace: csa_compress_decode_workspace_size() bytes (split-K partial
 * projections of the batch).
 * --------------------------------------------------------------------- */
int64_t csa_compress_decode_state_floats(const csa_geom* g);
size_t csa_compress_decode_workspace_size(const csa_geom* g, csa_dtype dtype, int B, int d);
csa_status csa_compress_decode(const csa_geom* g, csa_dtype dtype, const void* h,
                               const int64_t* pos, int B, int d, const void* W_aKV,
                               const void* W_bKV, const void* W_aZ, const void* W_bZ,
                               const float* bias, const float* gain, float* state,
                               csa_dtype out_dtype, void* E_cache, int64_t ldE, void* workspace,
                               size_t ws_bytes, csa_stream_t stream);

/* ---------------------------------------------------------------------
 * csa_index_topk - lightning indexer and top-k selection.
 * [EL] "CSA" Eqs 13-17; [SY] 03 index-score formula:
 *   I[q, s] = sum_h w[q,h] * ReLU(qI[q,h,:] . KI[seq, s, :]),  s < n_vis(q)
 *   n_vis(q) = min(floor((pos[q] + vis_offset)/m), n_entries[seq_of_q[q]]).
 * Keeps k_eff = min(k, n_vis) entries with the largest I; equal scores keep
 * the lower s. Output row q lists the kept s in ascending order, padded
 * with -1.
 *   qI        [Q, H_I, c_I] dtype (F32 or BF16)
 *   w         [Q, H_I] FP32
 *   KI        [nseq, ldK, c_I] dtype (queries whose seq_of_q is outside
 *             [0, nseq) see no entries)
 *   seq_of_q  [Q] int32, pos [Q] int64, n_entries [nseq] int64 (device)
 *   idx_out   [Q, k] int32
 *   scores_dbg [Q, ldK] FP32 or NULL: when given, the kernel's FP32 scores
 *             for s < n_vis(q) (other slots untouched) - a diagnostic.
 * 1 <= k <= CSA_MAX_TOPK; c_I a multiple of 16, <= 256; H_I <= 128.
 * n_vis is also clipped to ldK.
 * workspace: csa_index_topk_workspace_size() bytes.
 * --------------------------------------------------------------------- */
size_t csa_index_topk_workspace_size(int Q, int64_t ldK, int k);
csa_status csa_index_topk(const csa_geom* g, csa_dtype dtype, const void* qI, const float* w,
                          const void* KI, int64_t ldK, int nseq, const int32_t* seq_of_q,
                          const int64_t* pos, const int64_t* n_entries, int Q, int H_I,
                          int c_I, int k, int32_t* idx_out, float* scores_dbg,
                          void* workspace, size_t ws_bytes, csa_stream_t stream);

/* ---------------------------------------------------------------------
 * csa_index_scores - the lightning indexer's scores alone, without the
 * selection (the same equation, arguments and visibility as csa_index_topk).
 *   scores    [Q, ld_scores] FP32, ld_scores >= ldK: I[q, s] for
 *             s < n_vis(q); slots s >= n_vis(q) are left untouched.
 * The scores are bit-identical to the ones csa_index_topk selects from.
 * No workspace. Errors as for csa_index_topk.
 * --------------------------------------------------------------------- */
csa_status csa_index_scores(const csa_geom* g, csa_dtype dtype, const void* qI, const float* w,
                            const void* KI, int64_t ldK, int nseq, const int32_t* seq_of_q,
                            const int64_t* pos, const int64_t* n_entries, int Q, int H_I,
                            int c_I, float* scores, int64_t ld_scores, csa_stream_t stream);

/* ---------------------------------------------------------------------
 * csa_index_topk_noalloc - csa_index_topk without a caller workspace.
 * (An interface addition of this library; the pages have no counterpart.)
 * For callers that cannot allocate device memory around the call - code
 * running inside a memory arena that forbids outside allocations, or a
 * serving loop that must not allocate - the scores and top-k candidates
 * live in one fixed device buffer of CSA_NOALLOC_SCRATCH_BYTES compiled into
 * the library (every GPU that loads the library holds it until the process
 * exits). Arguments and results are those of csa_index_topk.
 *   - Returns CSA_ERR_TOO_LARGE, launching nothing, when
 *     csa_index_topk_workspace_size(Q, ldK, k) exceeds the buffer.
 *   - The first call on each device looks up the buffer's device address
 *     (with that device current); make that first call before any stream
 *     capture.
 *   - Allocates nothing: no cudaMalloc, no cudaFree, no allocating library
 *     routine.
 *   - Every call shares the one buffer, which keeps the last call's
 *     contents; nothing in it needs to start at zero (each value read is
 *     written earlier in the same call). Calls that overlap on the GPU
 *     (other streams, other host threads) race on the buffer: serialise
 *     them.
 * --------------------------------------------------------------------- */
#define CSA_NOALLOC_SCRATCH_BYTES (8u << 20)
csa_status csa_index_topk_noalloc(const csa_geom* g, csa_dtype dtype, const void* qI,
                                  const float* w, const void* KI, int64_t ldK, int nseq,
                                  const int32_t* seq_of_q, const int64_t* pos,
                                  const int64_t* n_entries, int Q, int H_I, int c_I, int k,
                                  int32_t* idx_out, float* scores_dbg, csa_stream_t stream);

/* ---------------------------------------------------------------------
 * csa_attend - shared-KV multi-query core attention over the selected
 * entries plus the sliding window, with one softmax and a sink.
 * [EL] "CSA" Eqs 18-19, "Shared attention details" (Sec 2.3.3, Eq 27);
 * [SY] 03; [CA] Sec 1 (one normalisation over window, compressed and sink).
 * For query q (sequence b = seq_of_q[q], position p = pos[q]) and head h:
 *   qh  = RoPE_p(RMSNorm(q[q,h,:]) * q_gain)
 *   J   = { E[b, idx[q,j]] : idx[q,j] >= 0 }  U  { win row of position j :
 *         max(0, p - n_win + 1) <= j <= p }
 *   l_j = qh . k_j / sqrt(c)
 *   o   = sum_j exp(l_j) k_j / (exp(sink[h]) + sum_j exp(l_j))
 *   O[q,h,:] = o with its last rope_dims dims rotated by -p.
 *   q     [Q, H_q, c] q_dtype (F32 or BF16); O [Q, H_q, c] q_dtype
 *   q_gain [c] FP32 or NULL (ones); sink [H_q] FP32
 *   E     [nseq, ldE, c] kv_dtype (F32, BF16, or mixed rows); queries whose
 *         seq_of_q is outside [0, nseq) produce zeros
 *   idx   [Q, k] int32, entries < n_entries[b] or -1 (slots holding -1 or
 *         an index >= ldE are skipped)
 *   win   [nseq, ldW, c] kv_dtype (F32 or BF16), rows already prepared
 *         (csa_rmsnorm_rope); row of position j = j (win_ring = 0, ldW > p)
 *         or j mod n_win (win_ring = 1, ldW >= n_win).
 * workspace: csa_attend_workspace_size() bytes, currently 0 for every
 * shape (the kernels keep their partial results on chip); callers may pass
 * NULL with ws_bytes = 0.
 * Results for a query do not depend on the other queries of the call while
 * Q < CSA_ATTEND_INVARIANT_Q (one thread-block cluster per query, split
 * boundaries fixed by k and n_win alone); larger calls run one CTA per
 * query, whose accumulation order differs (results agree within the
 * attention tolerance, not bit for bit).
 * --------------------------------------------------------------------- */
#define CSA_ATTEND_INVARIANT_Q 1024
size_t csa_attend_workspace_size(int Q, int H_q, int c, int k, int n_win);
csa_status csa_attend(const csa_geom* g, csa_dtype q_dtype, csa_dtype kv_dtype, const void* q,
                      const float* q_gain, const float* sink, const void* E, int64_t ldE,
                      int nseq, const int64_t* n_entries, const int32_t* idx, int k, const void* win,
                      int64_t ldW, const int32_t* seq_of_q, const int64_t* pos, int Q, int H_q,
                      void* O, void* workspace, size_t ws_bytes, csa_stream_t stream);

/* ---------------------------------------------------------------------
 * hca_attend - dense variant ([EL] "HCA"; [SY] 03: every completed,
 * causally available entry is read, no indexer). Same as csa_attend with
 * J = { E[b, s] : s < n_vis(q) } U window, n_vis computed from g->m and
 * g->vis_offset and clipped to n_entries[b].
 * workspace: hca_attend_workspace_size() bytes (currently 0).
 * --------------------------------------------------------------------- */
size_t hca_attend_workspace_size(int Q, int H_q, int c, int64_t ldE, int n_win);
csa_status hca_attend(const csa_geom* g, csa_dtype q_dtype, csa_dtype kv_dtype, const void* q,
                      const float* q_gain, const float* sink, const void* E, int64_t ldE,
                      int nseq, const int64_t* n_entries, const void* win, int64_t ldW,
                      const int32_t* seq_of_q, const int64_t* pos, int Q, int H_q, void* O,
                      void* workspace, size_t ws_bytes, csa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* CSA_H_ */
