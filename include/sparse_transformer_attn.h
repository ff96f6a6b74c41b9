/*
 * sparse_transformer_attn.h - C ABI of libsparse_transformer_attn.so
 *
 * Causal self-attention restricted to the factorized patterns of the Sparse
 * Transformer, forward and backward, as block-sparse attention on NVIDIA B200
 * (sm_100a).
 *
 * The operation ("Sparse Transformer" milestone page, nlp-lineage, "The idea",
 * paragraph "The notation"): for every head and query position i,
 *     O_i = softmax(q_i K_{S_i}^T * scale) V_{S_i},   scale = 1/sqrt(d),
 * where S_i is the head's allowed key set; the softmax normalises over S_i
 * only ("Sparse Transformer", llm-arch-kb, section 2 Derivation, "Sparse
 * attention as an unnormalized form"). Positions are 0-indexed.
 *   strided ("Pattern A"): A1_i = { j : max(0, i-l) <= j <= i }
 *                           A2_i = { j <= i : (i-j) mod l == 0 }
 *   fixed   ("Pattern B"): A1_i = { j <= i : floor(j/l) == floor(i/l) }
 *                           A2_i = { j <= i : j mod l >= l-c }
 *   dense causal:          S_i  = { j <= i }   (the comparator)
 * Heads: split  - head h uses A1 when h is even, A2 when h is odd
 *                 (milestone page, "The idea": each pattern is split between
 *                 two heads);
 *        merged - every head uses A1 u A2.
 * The backward pass recomputes the attention matrix from the saved
 * log-sum-exp instead of storing it (milestone page, "The idea",
 * "Recomputation").
 *
 * Conventions for every call below:
 *  - Tensors are caller-owned device pointers, contiguous [B, H, T, d]
 *    row-major, 16-byte aligned, all of one dtype (st_dtype). LSE is float32
 *    [B, H, T], natural log. The library owns only st_layout objects.
 *  - fwd and bwd enqueue work on `stream` (a cudaStream_t passed as void*;
 *    NULL = legacy default stream); they never allocate, never synchronise,
 *    and return as soon as the work is queued.
 *  - scale <= 0 selects 1/sqrt(d).
 *  - Errors are returned as st_status; nothing is thrown across the ABI.
 *    Invalid arguments return ST_ERR_INVALID before any launch; shapes the
 *    kernels do not implement return ST_ERR_UNSUPPORTED before any launch.
 *  - Supported shapes: bf16 or fp16 with d = 64 (tensor-core path), float32
 *    with d = 32 or 64 (exact fp32 path). T must be a multiple of 128; l must
 *    divide T or be >= T; for the fixed pattern with l < T, c must divide 128
 *    and satisfy 1 <= c <= l.
 */
#ifndef SPARSE_TRANSFORMER_ATTN_H
#define SPARSE_TRANSFORMER_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ST_OK = 0,
  ST_ERR_INVALID = 1,        /* bad argument: null pointer, bad size, mismatch */
  ST_ERR_UNSUPPORTED = 2,    /* valid, but not implemented by these kernels    */
  ST_ERR_CUDA = 3,           /* a CUDA runtime/driver call failed              */
  ST_ERR_DEVICE_TIMEOUT = 4, /* a bounded on-device wait ran out               */
  ST_ERR_WORKSPACE = 5       /* workspace missing or too small                 */
} st_status;

typedef enum { ST_STRIDED = 0, ST_FIXED = 1, ST_DENSE_CAUSAL = 2 } st_pattern_kind;
typedef enum { ST_HEADS_SPLIT = 0, ST_HEADS_MERGED = 1 } st_head_mode;
/* ST_F16: IEEE half precision, for the 16-bit mixed precision of the
 * milestone page ("The idea"); it runs the same tensor-core kernels as bf16, with
 * P and dS rounded to fp16 instead of bf16 and fp32 accumulation. */
typedef enum { ST_F32 = 0, ST_BF16 = 1, ST_F16 = 2 } st_dtype;

/* Pattern of one attention layer. l is the stride / block length
 * ("Sparse Transformer", llm-arch-kb, section 2: l ~ sqrt(T)); c is the number
 * of summary positions per block (fixed pattern only, 1 <= c <= l; ignored
 * otherwise). head_mode is ignored for ST_DENSE_CAUSAL. */
typedef struct {
  int32_t kind;      /* st_pattern_kind */
  int32_t head_mode; /* st_head_mode    */
  int32_t T;
  int32_t l;
  int32_t c;
} st_pattern_desc;

/* Opaque, library-owned block layout of one pattern (host copy plus device
 * copy). */
typedef struct st_layout st_layout;

/* Builds the block layout of a pattern ("Sparse Transformer", llm-arch-kb,
 * section 3: the per-query key indices are precomputed and the attention is a
 * block-sparse matmul). Every head's set S_i is split into disjoint segments;
 * each segment lists, per 128-query tile, its live 128-key tiles (CSR) and,
 * per key tile, its live query tiles (CSC), with a FULL/PARTIAL flag and the
 * live-pair count of every tile. Segments read keys in natural order, in
 * summary order (the last c positions of every block, packed) or in residue
 * order (position p*l + r at row p of class r, view row r*W + p), so that
 * their tiles are dense. Residue classes of P = T/l rows are padded to W =
 * 128*ceil(P/128) rows, except in strided layouts with 8 <= P <= 64 and P
 * dividing 128, where W = P (128/P whole classes per 128-row tile). Tile t of
 * a view covers view rows 128t .. 128t+127.
 * The device copy is uploaded with cudaMemcpyAsync on `stream`; the call
 * synchronises that stream once before returning. Runs once per shape.
 * Returns ST_ERR_INVALID for T < 1, l < 1, c outside [1, l] (fixed), or an
 * unknown kind/mode; ST_ERR_CUDA if the upload fails (no layout returned). */
st_status st_pattern_layout(const st_pattern_desc* desc, st_layout** out, void* stream);

/* Same, host copy only (no CUDA call; usable without a GPU, e.g. to inspect
 * or export a layout). fwd/bwd reject a host-only layout with
 * ST_ERR_INVALID. */
st_status st_pattern_layout_host(const st_pattern_desc* desc, st_layout** out);

void st_layout_destroy(st_layout* layout);

/* Numbers of head classes (2 for split heads: even, odd; else 1) and of
 * segments per head class. */
st_status st_layout_counts(const st_layout* layout, int32_t* n_head_classes,
                           int32_t* n_segments);

/* Key/query views and the membership rule of one segment:
 * view 0 natural, 1 summary (keys only), 2 residue class. */
st_status st_layout_segment_info(const st_layout* layout, int32_t head_class, int32_t segment,
                                 int32_t* query_view, int32_t* key_view, int32_t* rule);

/* Exports one segment's tile lists, or with segment = -1 the plain
 * natural-order 128x128 tiling of the whole set S_{h,i} of the head class.
 * transpose = 0 gives CSR over query tiles (ptr has n_query_tiles+1 entries,
 * idx = key tile), transpose = 1 gives CSC over key tiles. Tiles are listed in
 * ascending index order. flags[t] = 0 FULL (all 128x128 pairs live), 1
 * PARTIAL; live[t] = number of live pairs. sizes_inout[0] / [1] give the
 * capacities of ptr and of idx/flags/live; on return they hold the sizes
 * needed. Any output pointer may be NULL (size query). Returns ST_ERR_INVALID
 * for a bad head class or segment, ST_ERR_WORKSPACE if a capacity is short
 * (sizes are still written). */
st_status st_layout_export(const st_layout* layout, int32_t head_class, int32_t segment,
                           int32_t transpose, int32_t* ptr, int32_t* idx, uint8_t* flags,
                           int32_t* live, int64_t* sizes_inout);

/* Live pairs of one head of the class (sum over i of |S_i|). */
st_status st_layout_nnz(const st_layout* layout, int32_t head_class, int64_t* nnz);

/* Natural rows (positions t) of one head class that the 16-bit backward
 * treats in a given way, ascending. list 0: dQ rows accumulated in fp32
 * (several (key tile, query tile) pairs write them); 1: dK, dV rows
 * accumulated in fp32; 2: dQ rows no pair writes (queries with an empty set:
 * their gradient is zero and is zero-filled); 3: dK, dV rows no unit writes
 * (keys in no query's set, zero-filled). Rows in no list are written
 * directly in 16 bits. count_inout gives the capacity of rows (rows may be
 * NULL: size query) and returns the number of rows. Host data only: works on
 * layouts from st_pattern_layout_host. ST_ERR_INVALID for a bad head class or
 * list, ST_ERR_WORKSPACE if the capacity is short (the count is still
 * written). */
st_status st_layout_rows(const st_layout* layout, int32_t head_class, int32_t list,
                         int32_t* rows, int64_t* count_inout);

/* Forward: O and LSE for all B*H heads ("Sparse Transformer" milestone page,
 * nlp-lineage, "The idea", "The notation": O_i = softmax(q_i K_{S_i}^T / sqrt(d))
 * V_{S_i}, normalised over S_i only, llm-arch-kb section 2, "Sparse attention
 * as an unnormalized form"). Head h = index within H of the
 * [B, H, T, d] tensors (split mode picks A1/A2 from its parity). Rows with an
 * empty set get O = 0 and LSE = -inf. For a strided merged layout the call
 * runs two passes (natural-order window keys, then residue-order strided
 * keys) and merges them by log-sum-exp in place in o and lse. On the bf16
 * path each call takes one of the layout's 64 work counters in turn: at most
 * 64 forward calls of one layout may be in flight at the same time (on
 * different streams, or in concurrently replayed graphs). */
st_status st_sparse_attn_fwd(const st_layout* layout, st_dtype dtype, int32_t B, int32_t H,
                             int32_t T, int32_t d, float scale, const void* q, const void* k,
                             const void* v, void* o, float* lse, void* stream);

/* Bytes of device workspace st_sparse_attn_bwd needs for these sizes. */
st_status st_sparse_attn_bwd_workspace(const st_layout* layout, st_dtype dtype, int32_t B,
                                       int32_t H, int32_t T, int32_t d, size_t* bytes);

/* Backward ("Sparse Transformer" milestone page, nlp-lineage, "The idea",
 * "Recomputation": the attention matrix is rebuilt from the saved LSE rather
 * than stored): dQ, dK, dV (dtype of the inputs, fp32 accumulation) from Q, K,
 * V, the forward's O and LSE, and the upstream gradient dout. P is recomputed
 * as exp(s - LSE) on live tiles; D_i = dout_i . O_i. The workspace (device
 * memory, at least st_sparse_attn_bwd_workspace bytes, 256-byte aligned) is
 * overwritten; it holds D, the fp32 accumulators, a work counter and the
 * prologue's per-block maxima of |dout|. Returns ST_ERR_WORKSPACE if it is
 * missing or too small. On the 16-bit path dV is formed from P and dout in
 * fp16 (dout times a power of two chosen from its largest magnitude), and
 * rows with several contributions are summed by fp32 reduce-adds whose order
 * varies: results are not bitwise reproducible from run to run (within one
 * rounding step of the output type). */
st_status st_sparse_attn_bwd(const st_layout* layout, st_dtype dtype, int32_t B, int32_t H,
                             int32_t T, int32_t d, float scale, const void* q, const void* k,
                             const void* v, const void* o, const float* lse, const void* dout,
                             void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes,
                             void* stream);

/* Head-range forms ("Sparse Transformer", llm-arch-kb, section 2, "How the
 * two patterns are combined": the strided pattern on some heads and the fixed
 * pattern on the rest, in equal proportion). They compute exactly what
 * st_sparse_attn_fwd / st_sparse_attn_bwd compute, for heads h_begin ..
 * h_begin + h_count - 1 of tensors with H heads, and leave every other head's
 * rows of o, lse, dq, dk, dv untouched. Head indices stay global: a split
 * layout still gives head h the set of its parity. Mixed heads are one call
 * per layout on disjoint ranges; alternating patterns across layers is one
 * layout per layer. Tensors, workspace size and errors are those of the
 * full-range calls; ST_ERR_INVALID if the range is empty or leaves [0, H). */
st_status st_sparse_attn_fwd_heads(const st_layout* layout, st_dtype dtype, int32_t B,
                                   int32_t H, int32_t h_begin, int32_t h_count, int32_t T,
                                   int32_t d, float scale, const void* q, const void* k,
                                   const void* v, void* o, float* lse, void* stream);
st_status st_sparse_attn_bwd_heads(const st_layout* layout, st_dtype dtype, int32_t B,
                                   int32_t H, int32_t h_begin, int32_t h_count, int32_t T,
                                   int32_t d, float scale, const void* q, const void* k,
                                   const void* v, const void* o, const float* lse,
                                   const void* dout, void* dq, void* dk, void* dv,
                                   void* workspace, size_t ws_bytes, void* stream);

/* Backward pass for callers that cannot allocate device memory. The paper
 * has no counterpart: this is a deployment convenience of this library.
 * Some callers cannot call cudaMalloc or keep a workspace between calls
 * (a plugin whose host application owns every device allocation, or a
 * latency-critical path that must not allocate). This entry point computes
 * exactly what st_sparse_attn_bwd computes, with the same arguments except
 * the workspace: its scratch is a fixed 64 MiB array of library-owned device
 * memory, held until the process exits by every GPU where the library's
 * device code is loaded: under CUDA's default lazy module loading, a GPU on
 * which this entry point has been called; with CUDA_MODULE_LOADING=EAGER,
 * every GPU on which the process creates a context. It never allocates.
 *  - Limit: st_sparse_attn_bwd_workspace bytes for these sizes must not
 *    exceed 64 MiB (bf16: B*H*T*(4 + 12*d) + 4352 bytes, each part rounded
 *    up to 256 bytes); larger calls return ST_ERR_WORKSPACE before any
 *    launch. A layout built on another device than the current one returns
 *    ST_ERR_INVALID before the array is touched.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture.
 *  - All calls on a device share the one array, and it keeps the last call's
 *    contents (each call re-zeroes what must start at zero). Calls whose GPU
 *    work overlaps (other streams, other host threads) race on it and give
 *    wrong gradients: serialise them. */
st_status st_sparse_attn_bwd_noalloc(const st_layout* layout, st_dtype dtype, int32_t B, int32_t H,
                                     int32_t T, int32_t d, float scale, const void* q,
                                     const void* k, const void* v, const void* o,
                                     const float* lse, const void* dout, void* dq, void* dk,
                                     void* dv, void* stream);

/* Synchronises `stream`, then returns and clears the device-side status word
 * of the current device: ST_ERR_DEVICE_TIMEOUT after a kernel's bounded wait
 * ran out, ST_ERR_UNSUPPORTED if the backward kernel found its shared memory
 * misaligned (it then computes nothing); ST_OK otherwise. ST_ERR_CUDA if the
 * sync fails. */
st_status st_last_device_status(void* stream);

/* Upper bound, in nanoseconds, of every on-device wait of later launches
 * (default 2e9), process-wide: it applies to launches from every host thread
 * (the setting is atomic). 0 restores the default. A wait that runs out sets
 * the status word and makes the kernel return early. For tests of the timeout
 * path only, force_timeout != 0 makes the next bf16 / fp16 forward launch, from
 * whichever thread comes first, skip the loads of its first key tile so its
 * waits run out on purpose (the GPU stays usable). */
st_status st_set_wait_limit(uint64_t ns, int32_t force_timeout);

/* Kernel launches one fwd / bwd call makes with this layout and dtype (the
 * forward runs one launch per pass; the backward a prologue, its main
 * kernel(s) and, for bf16, an epilogue). */
st_status st_layout_launches(const st_layout* layout, st_dtype dtype, int32_t* fwd_launches,
                             int32_t* bwd_launches);

/* Benchmark instrumentation. enable != 0 creates (once) four pairs of CUDA
 * events on the current device; from then on every fwd call records pair 0
 * around its attention launches, and every bwd call records pair 1 around its
 * main attention kernel, pair 2 around its prologue and pair 3 around its
 * epilogue (16-bit path; the epilogue pair brackets nothing when no row
 * accumulates), on the call's stream. enable = 0 stops recording. Events are
 * created here, never inside fwd/bwd. Not thread-safe: one host thread may
 * time calls at a time. */
st_status st_kernel_timing(int32_t enable);

/* Milliseconds between the pair of events of the latest call of `kernel`
 * (0 = forward attention launches, 1 = backward main kernel, 2 = backward
 * prologue, 3 = backward epilogue); synchronises on that call's stop event.
 * ST_ERR_INVALID if timing is off or nothing ran. */
st_status st_kernel_elapsed_ms(int32_t kernel, float* ms);

/* Static description of a status code. */
const char* st_status_string(st_status status);

/* Library version, "major.minor.patch". */
const char* st_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SPARSE_TRANSFORMER_ATTN_H */
