/*
 * bsa.h -- C ABI of the B200 block-sparse attention library: the host
 * pattern builder, the forward, and for the same patterns the backward pass,
 * a decode step over a KV cache and content-based top-k block selection.
 *
 * The forward computes O = softmax(scale * Q K^T) V in which every query
 * row's softmax covers only the key blocks that its block row selects
 * ("Block Sparse Attention with Log-Linear Complexity", section 3.3: the
 * denominator sums only over the connected K blocks; unconnected positions
 * carry weight 0).  The block selection is a block-CSR built on the host
 * ("precompute the index table on the CPU before the launch", section 3.2 of
 * the same article).
 *
 * Conventions for every entry point:
 *  - The caller owns all memory.  The library never allocates device memory
 *    and never synchronises a stream.
 *  - Argument errors are reported synchronously by the return value, with
 *    nothing launched and nothing written.
 *  - Q, K, V, O are bf16, [B, H, N, d] contiguous (row-major, d fastest);
 *    LSE is fp32 [B, H, N].  Block-CSR rows are head-major: row h*M + i is
 *    block row i of head h, M = N / block_size; the same pattern applies to
 *    every batch entry b.
 */
#ifndef BSA_H
#define BSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes returned by every entry point. */
typedef enum {
  BSA_OK = 0,
  BSA_ERR_INVALID_ARG = -1,      /* null pointer, non-positive size, N % block_size != 0, ... */
  BSA_ERR_UNSUPPORTED = -2,      /* a legal value this build has no kernel for (d, block_size, M) */
  BSA_ERR_BUFFER_TOO_SMALL = -3, /* an output buffer cannot hold the result */
  BSA_ERR_BAD_PATTERN = -4,      /* a block-CSR violates the invariants listed at bsa_validate_pattern */
  BSA_ERR_CUDA = -5              /* a CUDA runtime/driver call failed; cudaGetLastError() has the cause */
} bsa_status;

/* Pattern kinds. */
typedef enum {
  /* "Block Sparse Attention with Log-Linear Complexity", sections 2.3 and 3.1:
   * local blocks |i-j| <= local_radius, log-stride blocks i +/- 2^k for
   * k = 0..log_kmax (block units), and global anchor columns (anchors[]; the
   * article names start, middle and end: 0, M/2, M-1).  Columns outside
   * [0, M) are dropped. */
  BSA_LOGLINEAR = 0,
  /* SparseFlashAttention article, "Local + Global" / "Block-Sparse": band
   * |i-j| <= local_radius, and every anchor block is a full row (it sees all
   * blocks) and a full column (all blocks see it). */
  BSA_LOCAL_GLOBAL = 1,
  /* RTX 4090 article, "core implementation logic" step 1: each (h, i, j) kept
   * with probability p, drawn from the counter-based SplitMix64 stream of
   * `seed` (output number key+1, key = (h*M + i)*M + j, u = top 53 bits /
   * 2^53, kept iff u < p); the diagonal is always kept. */
  BSA_BERNOULLI = 2,
  /* SparseFlashAttention article, "sparse pattern configuration examples"
   * (sliding_window: window and dilation "like a dilated convolution"),
   * taken at block level: column j is kept when |i-j| <= local_radius and
   * (i-j) is a multiple of `dilation` (the diagonal always is). */
  BSA_SLIDING_WINDOW = 3,
  /* SparseFlashAttention article, same examples (bigbird: random blocks,
   * block size, global tokens), with the three kinds of connections that
   * "Block Sparse Attention with Log-Linear Complexity", section 2.2, lists for
   * BigBird: a local window (|i-j| <= local_radius), global blocks (anchors:
   * full rows and full columns, as for BSA_LOCAL_GLOBAL) and `num_random`
   * random columns per (h, i): draw r = 0..num_random-1 takes output number
   * key+1 of the SplitMix64 stream of `seed` with key = (h*M + i)*num_random + r,
   * u = top 53 bits / 2^53, column floor(u*M); repeats merge. */
  BSA_BIGBIRD = 4
} bsa_kind;

/* Pattern description (caller-owned; anchors points to n_anchors ints). */
typedef struct {
  int32_t kind;          /* bsa_kind */
  int32_t M;             /* block rows = block columns, >= 1 */
  int32_t H;             /* heads, >= 1 (LOGLINEAR / LOCAL_GLOBAL repeat one head's rows) */
  int32_t local_radius;  /* LOGLINEAR: usually 1; LOCAL_GLOBAL: band half-width w, >= 0 */
  int32_t log_kmax;      /* LOGLINEAR: strides 2^k for k = 0..log_kmax, 0 <= log_kmax <= 30 */
  int32_t n_anchors;     /* number of entries in anchors, >= 0 */
  const int32_t* anchors;/* LOGLINEAR: anchor columns; LOCAL_GLOBAL: full rows and columns;
                            values outside [0, M) are ignored */
  double p;              /* BERNOULLI keep probability in [0, 1] */
  uint64_t seed;         /* BERNOULLI stream seed */
  int32_t causal;        /* 0 or 1: keep only columns j <= i */
  int32_t dilation;      /* SLIDING_WINDOW: keep j with (i-j) % dilation == 0, >= 1 */
  int32_t num_random;    /* BIGBIRD: random columns drawn per block row, >= 0 */
} bsa_pattern_desc;

/*
 * bsa_build_pattern -- host-only, integer work only.
 *
 * Builds the block-CSR of `desc` over H*M rows: row_ptr[H*M+1] and the
 * columns of every row in ascending order without repeats.
 * Two-call use: with row_ptr == NULL and col_idx == NULL only *nnz_out is
 * written (the number of stored blocks over all heads).  Otherwise row_ptr
 * must hold H*M+1 ints and col_idx `cap` ints; if cap < nnz the call returns
 * BSA_ERR_BUFFER_TOO_SMALL and writes only *nnz_out.
 * Returns BSA_ERR_INVALID_ARG for a null desc/nnz_out, M < 1, H < 1, an
 * unknown kind, a negative radius, log_kmax outside [0, 30], p outside
 * [0, 1], n_anchors < 0 or anchors == NULL with n_anchors > 0, causal not
 * 0/1, dilation < 1 (SLIDING_WINDOW), num_random < 0 (BIGBIRD), or an nnz
 * that does not fit int32.  BERNOULLI and BIGBIRD draw every head on its
 * own; the other kinds repeat one head's rows.
 */
int bsa_build_pattern(const bsa_pattern_desc* desc, int32_t* row_ptr, int32_t* col_idx,
                      int64_t cap, int64_t* nnz_out);

/*
 * bsa_validate_pattern -- host-only check of a block-CSR held in host memory.
 *
 * Checks: row_ptr[0] == 0; row_ptr non-decreasing; row_ptr[H*M] <= col_cap
 * (else BSA_ERR_BUFFER_TOO_SMALL); every column in [0, M); columns strictly
 * ascending within a row; with causal == 1 every column j of block row i has
 * j <= i.  Returns BSA_OK or BSA_ERR_BAD_PATTERN (BSA_ERR_INVALID_ARG for
 * null pointers or non-positive H, M).
 */
int bsa_validate_pattern(const int32_t* row_ptr, const int32_t* col_idx, int64_t col_cap,
                         int32_t H, int32_t M, int32_t causal);

/*
 * bsa_forward -- the block-sparse attention forward on the current CUDA
 * device, enqueued on `stream` (a cudaStream_t; NULL = legacy default).
 *
 * For batch b, head h and query token q of block row r = q / block_size:
 *   keys(q) = tokens of the blocks col_idx[row_ptr[h*M+r] .. row_ptr[h*M+r+1])
 *             minus the tokens k > q when causal == 1;
 *   O[b,h,q,:] = sum_k softmax_k(scale * Q[b,h,q,:] . K[b,h,k,:]) V[b,h,k,:]
 *   LSE[b,h,q] = ln sum_k exp(scale * Q[b,h,q,:] . K[b,h,k,:])   (natural log)
 *   An empty keys(q) gives O = 0 and LSE = -inf.
 * Inputs bf16, products and sums in fp32 on the tensor cores, softmax
 * statistics in fp32, O rounded to bf16 (nearest even).
 *
 * Q, K, V, O: device pointers, bf16 [B,H,N,d] contiguous, 16-byte aligned.
 * LSE: device pointer, fp32 [B,H,N], 16-byte aligned.  O and LSE must not
 * overlap the inputs.
 * row_ptr: device int32 [H*M+1]; col_idx: device int32 [row_ptr[H*M]].
 * The columns of a row may come in any order; a repeated column counts once.
 * Columns outside [0, M) are skipped and flagged in the device status word
 * (bsa_device_status).  row_ptr must be non-decreasing and col_idx must hold
 * row_ptr[H*M] entries: the call does not read the CSR on the host (use
 * bsa_validate_pattern there).
 * Supported: d in {64, 128}; block_size in {32, 64, 128}; N % block_size == 0;
 * 1 <= M <= 4096; B*H <= 2^31-1.  Else BSA_ERR_INVALID_ARG /
 * BSA_ERR_UNSUPPORTED, nothing launched.  A failed launch returns BSA_ERR_CUDA.
 * The call returns without synchronising.
 */
int bsa_forward(const void* Q, const void* K, const void* V,
                const int32_t* row_ptr, const int32_t* col_idx,
                int B, int H, int N, int d, int block_size, float scale, int causal,
                void* O, float* LSE, void* stream);

/*
 * bsa_forward_ws -- bsa_forward with a workspace for chunked tiles.
 *
 * The kernel's unit of work is a tile of 128 query rows walking the union of
 * its block rows' columns.  When one tile's walk is longer than two even
 * shares of the whole launch per tile slot (a global row on a small problem,
 * say), its walk is cut into chunks that run as separate units; each chunk
 * leaves its unnormalised O and its (max, sum) statistics in the workspace
 * and the last chunk of the tile to finish merges them, weighting chunk c by
 * exp(m_c - max_c m_c) ("split long rows into kv-chunks"; the merged softmax
 * is the one of section 3.3 of "Block Sparse Attention with Log-Linear
 * Complexity" over the union of the chunks' keys).  The result is the same
 * function as bsa_forward's, up to fp32 rounding.
 *
 * Arguments as bsa_forward, plus workspace: caller-owned device memory,
 * 16-byte aligned, of up to bsa_forward_workspace_bytes(d) bytes (a smaller
 * one allows fewer chunks; below one chunk, or NULL, no tile is cut, which is
 * bsa_forward).  Its contents need not be initialised and are overwritten;
 * one workspace must not serve two launches that may run at the same time.
 * Nothing is allocated and nothing synchronised.  Errors as bsa_forward;
 * BSA_ERR_INVALID_ARG also for a misaligned workspace.
 */
size_t bsa_forward_workspace_bytes(int d);  /* 0 for an unsupported d */
int bsa_forward_ws(const void* Q, const void* K, const void* V,
                   const int32_t* row_ptr, const int32_t* col_idx,
                   int B, int H, int N, int d, int block_size, float scale, int causal,
                   void* O, float* LSE, void* workspace, size_t workspace_bytes, void* stream);

/* Bits of the device status word. */
#define BSA_STATUS_TIMEOUT     0x1u  /* a bounded wait inside the kernel gave up */
#define BSA_STATUS_BAD_COLUMN  0x2u  /* a column index outside [0, M) was skipped */
#define BSA_STATUS_BAD_ROW_PTR 0x4u  /* row_ptr[i] < 0 or row_ptr[i+1] < row_ptr[i] was seen; the row was treated as empty */
#define BSA_STATUS_BAD_SEQ_LEN 0x8u  /* bsa_decode: a seq_len outside [1, L]; that entry was treated as empty */
#define BSA_STATUS_INTERNAL    0x10u /* a kernel found its own work plan inconsistent and stopped; a library fault */

/*
 * Content-based top-k block selection (a pattern computed from Q and K on the
 * device).  The SparseFlashAttention article ("pattern generation", third
 * kind) chooses the Top-K positions by the similarity of Q and K; the RTX
 * 4090 article uses "dynamic sparsity, topk = 20%".  At block level:
 *   Qm[i, c] = (sum over the bs tokens t of block i of Q[t, c]) / bs, Km alike;
 *   s[i, j]  = sum over c of Qm[i, c] * Km[j, c];
 *   row i keeps its diagonal block and the top_k highest-scoring other
 *   allowed blocks (j != i; j <= i when causal), ties to the smaller j.
 * All arithmetic is fp64 in a fixed order (tokens, then c, ascending; each
 * product rounded on its own, no fused multiply-add), so that the selection
 * is reproducible.  One CSR row per (b*H + h, i): run the forward on the
 * result with the batch folded into the heads, [1, B*H, N, d].
 *
 * Row i holds 1 + min(top_k, i if causal else M - 1) columns, ascending, so
 * row_ptr is fixed by (BH, M, top_k, causal); bsa_topk_nnz gives the total.
 */

/* Total stored blocks of a top-k pattern; -1 for BH < 1, M < 1 or top_k < 0. */
int64_t bsa_topk_nnz(int BH, int M, int top_k, int causal);

/* Device workspace bytes bsa_topk_pattern needs (the fp64 block means of Q
 * and K): 2 * BH * (N / block_size) * d * 8; 0 for invalid sizes. */
size_t bsa_topk_workspace_bytes(int BH, int N, int d, int block_size);

/*
 * bsa_topk_pattern -- the selection above, enqueued on `stream`.
 *
 * Q, K: device bf16 [BH, N, d] contiguous (BH = B*H).  row_ptr: device int32
 * [BH*M+1]; col_idx: device int32 [bsa_topk_nnz(...)]; workspace: caller-owned
 * device memory of at least bsa_topk_workspace_bytes(...) bytes, 8-byte
 * aligned, which the call overwrites (it need not be zeroed).  Nothing is
 * allocated and nothing synchronised.
 * Supported: 1 <= d <= 256, block_size >= 1, N % block_size == 0,
 * 1 <= M <= 4096, top_k >= 0, causal 0/1, BH >= 1.  Else
 * BSA_ERR_INVALID_ARG / BSA_ERR_UNSUPPORTED with nothing launched;
 * BSA_ERR_BUFFER_TOO_SMALL for a short workspace; BSA_ERR_CUDA if a launch
 * fails.
 */
int bsa_topk_pattern(const void* Q, const void* K, int BH, int N, int d, int block_size,
                     int top_k, int causal, int32_t* row_ptr, int32_t* col_idx,
                     void* workspace, size_t workspace_bytes, void* stream);

/*
 * bsa_topk_pattern_static -- bsa_topk_pattern without a caller workspace and
 * without any allocation.  The pages have no counterpart: this is an
 * interface of this library only, for callers that must not allocate device
 * memory around the selection.
 *
 * The fp64 block means live in a scratch array of the library itself (a
 * file-scope __device__ array, 256-byte aligned, one copy per device) of
 * BSA_TOPK_STATIC_SCRATCH_BYTES.  Its address is looked up with
 * cudaGetSymbolAddress on the first call on each device (the current device
 * at the call), so make that first call before any stream capture on that
 * device.  The call makes no cudaMalloc, cudaFree or other allocating call.
 * The address is kept for the life of the process: after cudaDeviceReset (or
 * any reset of the device's primary context) it is stale, so do not call this
 * entry point again on that device in the same process.
 *
 * Arguments, layouts, results and the other errors are those of
 * bsa_topk_pattern (same kernels, same bits).  A request whose workspace,
 * bsa_topk_workspace_bytes(BH, N, d, block_size), exceeds
 * BSA_TOPK_STATIC_SCRATCH_BYTES (that is BH * M * d > 262144) returns
 * BSA_ERR_BUFFER_TOO_SMALL before any CUDA call, with nothing launched and
 * the outputs untouched; use bsa_topk_pattern with a workspace instead.
 * BSA_ERR_CUDA if the symbol lookup or a launch fails; BSA_ERR_UNSUPPORTED
 * for a device ordinal of 64 or more.
 *
 * Nothing needs to start at zero: neither the scratch (each call writes every
 * element it reads before reading it) nor row_ptr / col_idx.
 * Calls that overlap in time on one device -- on different streams, or from
 * host threads without an order between them -- share the one scratch array
 * and race; order them (one stream, or events).
 */
#define BSA_TOPK_STATIC_SCRATCH_BYTES (4u * 1024u * 1024u)
int bsa_topk_pattern_static(const void* Q, const void* K, int BH, int N, int d, int block_size,
                            int top_k, int causal, int32_t* row_ptr, int32_t* col_idx,
                            void* stream);

/*
 * bsa_transpose_pattern -- column-major copy of a block-CSR, for the
 * backward's dK/dV walk (host only, integer work).  For every (h, column j)
 * col_ptr[h*M + j] .. col_ptr[h*M + j + 1] indexes row_idx, the block rows
 * i that list j, ascending; a column repeated within a row counts once.
 * row_ptr [H*M+1], col_idx: host arrays of a CSR; col_ptr: host int32
 * [H*M+1]; row_idx: host int32 of capacity `cap` (at most row_ptr[H*M]
 * entries are written).  *nnz_out receives the entry count, also when it
 * exceeds cap (then BSA_ERR_BUFFER_TOO_SMALL, nothing written).
 * BSA_ERR_BAD_PATTERN for a decreasing row_ptr, row_ptr[0] != 0 or a column
 * outside [0, M); BSA_ERR_INVALID_ARG for null pointers or H, M < 1.
 */
int bsa_transpose_pattern(const int32_t* row_ptr, const int32_t* col_idx, int32_t H, int32_t M,
                          int32_t* col_ptr, int32_t* row_idx, int64_t cap, int64_t* nnz_out);

/* Device workspace bytes bsa_backward needs: D = dO . O per query row (fp32),
 * then per 128-row tile two costs and two positions of the heavy-first tile
 * orders (int32): 4*B*H*N + 16*B*H*ceil(N/128); 0 for invalid sizes. */
size_t bsa_backward_workspace_bytes(int B, int H, int N);

/*
 * bsa_backward -- gradients of bsa_forward: dQ, dK, dV.
 *
 * "Block Sparse Attention with Log-Linear Complexity" notes that the sparse
 * product falls back to dense work in the backward pass (section 4.2) and
 * trains with the pattern (section 5.3).  With P_qk = exp(scale q.k - LSE_q)
 * over the keys the forward allowed and D_q = dO_q . O_q:
 * dV_k = sum_q P dO_q; dS = P (dO_q . v_k - D_q); dQ_q = scale sum_k dS k_k;
 * dK_k = scale sum_q dS q_q.
 *
 * Q, K, V, O, dO: device bf16 [B, H, N, d] contiguous (O and LSE from
 * bsa_forward on the same inputs and pattern); LSE: device fp32 [B, H, N].
 * row_ptr / col_idx: the forward's block-CSR (device); col_ptr / row_idx: its
 * column-major copy from bsa_transpose_pattern (device).  dQ, dK, dV: device
 * bf16 [B, H, N, d], fully written.  workspace: device memory of at least
 * bsa_backward_workspace_bytes(B, H, N) bytes, 16-byte aligned (overwritten;
 * nothing in it needs to start at zero).  Enqueued on `stream` (five kernels:
 * D, the tile costs, the heavy-first tile orders, dK/dV, dQ); nothing
 * allocated or synchronised.
 * Supported: d in {64, 128}; block_size in {32, 64, 128}; N % 128 == 0;
 * M <= 4096; 16-byte aligned tensors.  Else BSA_ERR_INVALID_ARG /
 * BSA_ERR_UNSUPPORTED with nothing launched; BSA_ERR_BUFFER_TOO_SMALL for a
 * short workspace; BSA_ERR_CUDA if a launch fails.  Device-side checks set
 * BSA_STATUS_* bits read by bsa_backward_status.
 */
int bsa_backward(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                 const float* LSE, const int32_t* row_ptr, const int32_t* col_idx,
                 const int32_t* col_ptr, const int32_t* row_idx, int B, int H, int N, int d,
                 int block_size, float scale, int causal, void* dQ, void* dK, void* dV,
                 void* workspace, size_t workspace_bytes, void* stream);

/* bsa_backward_status -- as bsa_device_status, for the backward kernels' word. */
int bsa_backward_status(uint32_t* status, int clear);

/*
 * bsa_decode -- one decode step of block-sparse attention over a KV cache.
 *
 * "Block Sparse Attention with Log-Linear Complexity" keeps the KV cache in
 * the (B, H, N, D) layout of past_key_values (section 5.1) and claims the
 * pattern cuts cache traffic at inference (section 1).  For each (b, h), the
 * new token sits at position t = seq_len[b] - 1, in block row i = t /
 * block_size.  It attends to the cached tokens of the blocks j <= i listed
 * in CSR row i of head h: all block_size tokens of a block j < i, the tokens
 * i*block_size .. t of block i (blocks j > i hold no cached tokens yet and are
 * skipped).  O = sum softmax(scale * q.k) v; LSE = the natural log-sum-exp of
 * the scaled scores; no tokens gives O = 0 and LSE = -inf.  A row is a set
 * (repeated columns count once).
 *
 * q: bf16 [B, H, d]; k_new, v_new: bf16 [B, H, d], or both NULL; k_cache,
 * v_cache: bf16 [B, H, L, d] contiguous.  With k_new/v_new given the step
 * first writes them into cache row t of each (b, h) -- the append of the new
 * token -- and attends to them there; otherwise row t must already hold the
 * new token.  Rows after t are never read.  row_ptr int32 [H*M+1] and
 * col_idx int32: the forward's block-CSR over M = L / block_size block rows.
 * seq_len: device int32 [B], cached tokens including the new one, 1..L.
 * O: bf16 [B, H, d]; LSE: fp32 [B, H].  All pointers are caller-owned
 * device memory, 16-byte aligned (LSE 4-byte); the call is enqueued on
 * `stream` and allocates nothing.
 * Supported: d in {64, 128}; block_size in {32, 64, 128}; L % block_size ==
 * 0; M <= 4096.  Else BSA_ERR_INVALID_ARG / BSA_ERR_UNSUPPORTED with nothing
 * launched; BSA_ERR_CUDA if the launch fails.  Device-side checks (a
 * seq_len outside [1, L], a column outside [0, M), a decreasing row_ptr, a
 * timed-out wait) set BSA_STATUS_* bits read by bsa_decode_status.
 */
int bsa_decode(const void* q, const void* k_new, const void* v_new, void* k_cache,
               void* v_cache, const int32_t* row_ptr, const int32_t* col_idx,
               const int32_t* seq_len, int B, int H, int L, int d, int block_size,
               float scale, void* O, float* LSE, void* stream);

/* bsa_decode_status -- as bsa_device_status, for the status word the decode
 * kernel sets (BSA_STATUS_TIMEOUT, _BAD_COLUMN, _BAD_ROW_PTR, _BAD_SEQ_LEN). */
int bsa_decode_status(uint32_t* status, int clear);

/*
 * bsa_device_status -- read (and with clear != 0, reset) the status word of
 * the current device.  Synchronises the device.  Returns BSA_OK or
 * BSA_ERR_CUDA; *status receives an OR of BSA_STATUS_* bits accumulated by
 * the kernels since the last clear.
 */
int bsa_device_status(uint32_t* status, int clear);

/* Library version as an integer (major*10000 + minor*100 + patch). */
int bsa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BSA_H */
