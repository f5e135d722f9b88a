/*
 * llsa.h -- C ABI of the B200 (sm_100a) implementation of Log-linear Sparse
 * Attention (LLSA) for pixel-space diffusion transformers.
 *
 * The method (cited by page title and section):
 *   [LLSA] "Trainable Log-linear Sparse Attention for Efficient Diffusion
 *          Transformers" (CVPR 2026), technical summary page: §三 hierarchical
 *          top-K, §四 hierarchical KV enrichment and KV reweighting, §4.1
 *          sparse backward, §4.2 / Fig. 2 index reordering.
 *   [ART]  popular write-up of arXiv:2512.16615, §三 (hierarchical selection,
 *          weight = block size of the level) and §四 (sparse-index forward,
 *          CSR->CSC index transpose, reordering).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * * Tensors are caller-owned DEVICE buffers, contiguous, 16-byte aligned.
 *   Token tensors are [batch, heads, N, d] with N = height * width, element
 *   type `dtype` (bf16 or fp32).  Every call except llsa_reorder takes them in
 *   HIERARCHICAL token order (see llsa_reorder).
 * * Level l = 1..L holds n_l = N / B^l pooled tokens.  Index lists have
 *   K_L = min(K, n_L) entries per token at the coarsest level and
 *   K_l = min(K, K_{l+1} * B) at finer levels ([LLSA] §三).
 * * Level-packed buffers hold level 1 first, then level 2, ...; inside a level
 *   the layout is [batch*heads][n_l][...].  Sizes come from llsa_query_sizes:
 *     pyramid   fp32  [BH][n_l][d]         per level
 *     idx       int32 [BH][n_l][K_l]       per level, each list ascending
 *     offs      int32 [BH][n_l + 1]        per level (CSC offsets)
 *     qlist     int32 [BH][n_l * K_l]      per level (CSC query ids, ascending per key)
 * * The library allocates nothing and keeps no state between calls; calls are
 *   asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream).
 * * Host-detectable errors (bad shapes, NULL or misaligned pointers,
 *   unsupported sizes) return a status before anything is launched.  A
 *   launch failure returns LLSA_ERR_CUDA.  No exception crosses the ABI.
 * * Buffer sizes are queried with llsa_query_sizes (one call returns every
 *   size, the workspaces included); device-side timeouts are read with
 *   llsa_device_error.  The main entry points take no size arguments: their
 *   buffers must have the queried sizes.  LLSA_ERR_WORKSPACE is returned only
 *   by llsa_index_transpose_noalloc, whose scratch has a fixed size.
 * * Pooled tokens: pyrK / pyrV passed to the attention calls must be what
 *   llsa_pool wrote for the same k / v.  Level 1 is then the exact mean of
 *   the B key (value) rows it stands for, and the tensor-core kernels (bf16,
 *   d = 64, B = 16) use that identity: they form level-1 pooled logits and
 *   values from k / v themselves and do not read level 1 of pyrK / pyrV.  The
 *   CUDA-core kernels (every other problem) read it.  Levels >= 2 are read by
 *   both.
 */
#ifndef LLSA_H
#define LLSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Binary-compatible with cudaStream_t; no CUDA header needed to include this file. */
typedef struct CUstream_st* llsa_stream;

typedef enum {
  LLSA_OK = 0,
  LLSA_ERR_ARG = 1,          /* NULL pointer or invalid field */
  LLSA_ERR_SHAPE = 2,        /* image does not tile into sqrt(B)^L squares, or sizes overflow */
  LLSA_ERR_ALIGN = 3,        /* a buffer is not 16-byte aligned */
  LLSA_ERR_WORKSPACE = 4,    /* the fixed scratch of llsa_index_transpose_noalloc is too small */
  LLSA_ERR_CUDA = 5,         /* a CUDA launch or runtime call failed */
  LLSA_ERR_TIMEOUT = 6,      /* a bounded device-side wait gave up (see llsa_device_error) */
  LLSA_ERR_UNSUPPORTED = 7   /* valid problem outside what the kernels implement */
} llsa_status;

typedef enum { LLSA_BF16 = 0, LLSA_FP32 = 1 } llsa_dtype;

#define LLSA_MAX_LEVELS 12

typedef struct {
  int batch, heads;       /* independent (batch, head) slices */
  int height, width;      /* image size in pixels; N = height * width tokens */
  int d;                  /* head dimension (multiple of 8, at most 128) */
  int B;                  /* block size, a perfect square B = t * t, t >= 2 */
  int L;                  /* pooled levels, 1 <= L <= LLSA_MAX_LEVELS; height and width divisible by t^L */
  int K;                  /* top-K per level; K >= number of candidates keeps all of them */
  unsigned enrich_mask;   /* bit (l-1) set: level-l coarse K/V join the attention ([LLSA] §四) */
  float scale;            /* softmax scale; 0 selects 1/sqrt(d) */
  int dtype;              /* llsa_dtype of Q, K, V, O, dO, dQ, dK, dV */
} llsa_problem;

typedef struct {
  size_t tokens_bytes;              /* one [BH][N][d] tensor of `dtype` */
  size_t lse_bytes;                 /* fp32 [BH][N] */
  size_t pyramid_bytes;             /* one fp32 pyramid, levels 1..L */
  size_t idx_bytes;                 /* int32 index lists, all levels */
  size_t offs_bytes;                /* int32 CSC offsets, all levels */
  size_t qlist_bytes;               /* int32 CSC query ids, all levels */
  size_t transpose_scratch_bytes;   /* scratch for llsa_index_transpose */
  size_t bwd_workspace_bytes;       /* workspace for llsa_attn_bwd */
} llsa_sizes;

/* Human-readable name of a status. */
const char* llsa_status_string(llsa_status s);

/* Checks every field of *p; no launch.  LLSA_OK, LLSA_ERR_ARG, LLSA_ERR_SHAPE or
 * LLSA_ERR_UNSUPPORTED. */
llsa_status llsa_validate(const llsa_problem* p);

/* n[0..L] (tokens per level, n[0] = N) and Kl[0..L] (list length per level,
 * Kl[0] = 0).  Host memory, L+1 entries each. */
llsa_status llsa_level_sizes(const llsa_problem* p, int64_t* n, int64_t* Kl);

/* Byte sizes of every buffer the entry points take. */
llsa_status llsa_query_sizes(const llsa_problem* p, llsa_sizes* out);

/* Index reordering ([ART] §四; [LLSA] §4.2, Fig. 2).  Moves token rows between
 * raster order (row y*W + x) and hierarchical order: recursive sqrt(B) x sqrt(B)
 * tiles, row-major inside every tile and row-major over the top grid of
 * t^L x t^L squares, so that every aligned run of B^l hierarchical positions
 * is one t^l x t^l pixel square:
 *   hier(y,x) = (floor(y/t^L)*(W/t^L) + floor(x/t^L)) * B^L
 *             + sum_{l=1..L} ((floor(y/t^(l-1)) mod t)*t + floor(x/t^(l-1)) mod t) * B^(l-1).
 * in, out: [BH][N][d] of dtype; to_hier != 0 maps raster -> hierarchical,
 * 0 maps back.  in and out must not overlap. */
llsa_status llsa_reorder(const llsa_problem* p, const void* in, void* out, int to_hier, llsa_stream stream);

/* Hierarchical compression ([LLSA] §三): P_l[j] = mean of P_{l-1}[j*B .. j*B+B-1],
 * l = 1..L, P_0 = x.  x: hierarchical [BH][N][d] of dtype; pyramid: fp32, level
 * packed, pyramid_bytes.  Call once each for Q, K and V. */
llsa_status llsa_pool(const llsa_problem* p, const void* x, float* pyramid, llsa_stream stream);

/* Coarse-to-fine top-K selection ([LLSA] §三; [ART] §三).  Level L: every
 * level-L query token scores all n_L level-L keys.  Level l < L: query token a
 * scores only the B children of each pick of its parent floor(a/B) at level
 * l+1.  Score = pooled q . pooled k in fp32; the K_l best are kept (higher
 * score first, lower key id on equal scores) and stored ascending.
 * pyrQ, pyrK: pyramids from llsa_pool; idx: idx_bytes, all levels written. */
llsa_status llsa_select(const llsa_problem* p, const float* pyrQ, const float* pyrK, int32_t* idx,
                        llsa_stream stream);

/* One level of llsa_select: reads the level-(level+1) lists already in idx
 * (when level < L) and writes the level-`level` lists only. */
llsa_status llsa_select_level(const llsa_problem* p, int level, const float* pyrQ, const float* pyrK,
                              int32_t* idx, llsa_stream stream);

/* Sparse attention forward with hierarchical KV enrichment ([LLSA] §四;
 * [ART] §三, §四).  Fine query i (block a = floor(i/B)) attends to
 *   the B tokens of each level-1 block in S_1(a), logit scale * q.k, and
 *   for every level l set in enrich_mask the pooled tokens S_l(floor(i/B^l))
 *   of pyrK/pyrV, logit scale * q.P^K_l + ln(B^l)  (weight B^l).
 * Keys are gathered by index; no mask is built.
 * q, k, v: hierarchical [BH][N][d] of dtype; pyrK, pyrV: pyramids of K and V;
 * idx: from llsa_select; o: [BH][N][d] of dtype; lse: fp32 [BH][N], natural log
 * of the softmax denominator (with the weights). */
llsa_status llsa_attn_fwd(const llsa_problem* p, const void* q, const void* k, const void* v,
                          const float* pyrK, const float* pyrV, const int32_t* idx, void* o, float* lse,
                          llsa_stream stream);

/* Sparse index transpose, CSR -> CSC ([ART] §四; [LLSA] §4.1), every level:
 * per-key counts (warp-aggregated atomics), exclusive prefix sum into offs,
 * scatter of the query ids into qlist, each key's ids ascending.
 * scratch: transpose_scratch_bytes of device memory, contents ignored. */
llsa_status llsa_index_transpose(const llsa_problem* p, const int32_t* idx, int32_t* offs, int32_t* qlist,
                                 void* scratch, llsa_stream stream);

/* llsa_index_transpose without a scratch argument.  The pages have no
 * counterpart to this entry point; it exists for callers that cannot obtain
 * device memory at the point where they run the transpose -- for example a
 * plug-in whose host framework owns every device allocation and exposes no
 * allocator to it, or a latency-critical loop that must never call
 * cudaMalloc (which can synchronize the device).  Those callers still pass
 * idx, offs and qlist, but no scratch: the scratch lives in a fixed 16 MiB
 * device array inside this library (every GPU that loads the library holds
 * it until the process exits).  A problem whose transpose needs more than
 * that (transpose_scratch_bytes > 16 MiB) is rejected with
 * LLSA_ERR_WORKSPACE before anything is launched.  Nothing is allocated:
 * no cudaMalloc, no cudaFree.
 * Every call looks up the array's device address on the current device
 * (cudaGetSymbolAddress, a host-side lookup that launches nothing), so a
 * device reset between calls leaves no stale address behind.  The first call
 * on a device may load this library's device code there; make it before any
 * stream capture.  All calls share the one array and it
 * keeps whatever the last call left there (the parts that must start at zero
 * are cleared by every call), so two calls whose work overlaps on the GPU --
 * on different streams, or from different threads -- race and must be
 * serialized by the caller.  Results are identical to llsa_index_transpose. */
llsa_status llsa_index_transpose_noalloc(const llsa_problem* p, const int32_t* idx, int32_t* offs,
                                         int32_t* qlist, llsa_stream stream);

/* Sparse attention backward ([LLSA] §4.1), index lists held fixed.  With
 * P = exp(z - lse) and D_i = dO_i . o_i:  dq_i = scale * sum_j P_ij (dO_i.v_j - D_i) k_j;
 * fine keys gather their queries through the level-1 CSC lists (offs, qlist);
 * pooled keys accumulate into fp32 level gradients that are sent back to the
 * B^l tokens they average (dk_t += dPK_l[floor(t/B^l)] / B^l, the same for v).
 * Pooled Q receives no gradient.  o, lse: from llsa_attn_fwd; dO: upstream
 * gradient; dq, dk, dv: [BH][N][d] of dtype, fully written; workspace:
 * bwd_workspace_bytes of device memory, contents ignored. */
llsa_status llsa_attn_bwd(const llsa_problem* p, const void* q, const void* k, const void* v,
                          const void* o, const void* dO, const float* lse, const float* pyrK,
                          const float* pyrV, const int32_t* idx, const int32_t* offs, const int32_t* qlist,
                          void* dq, void* dk, void* dv, void* workspace, llsa_stream stream);

/* Which kernels llsa_attn_fwd and llsa_attn_bwd run for *p (host only, no
 * launch): *fwd_tc / *bwd_tc = 1 for the tensor-core kernels (tcgen05 /
 * TMEM, bf16, d = 64, B = 16, within the sizes they support), 0 for the
 * CUDA-core kernels.  Either pointer may be NULL. */
llsa_status llsa_attn_paths(const llsa_problem* p, int* fwd_tc, int* bwd_tc);

/* Number of CUDA kernels this library has launched in this process so far
 * (all entry points, all streams); for accounting in benchmarks. */
uint64_t llsa_kernel_launches(void);

/* Waits for `stream`, then reads and clears the device-side error word that
 * bounded waits inside the kernels set when they give up.  *code = 0 when no
 * wait gave up; returns LLSA_ERR_TIMEOUT when one did.  There is one word
 * per device, shared by every stream and thread of the process: a code
 * cannot be attributed to one stream, and a read clears it for all. */
llsa_status llsa_device_error(llsa_stream stream, int* code);

/* Self-test of the timeout path of the bounded device waits: launches one
 * thread on `stream` that waits, with the same bounded wait the pipelined
 * kernels use, on an mbarrier phase that nothing completes (arrive = 0) or
 * that it completed itself first (arrive = 1).  When the wait gives up after
 * limit_us microseconds the device error word is set to `code`, so that the
 * next llsa_device_error returns LLSA_ERR_TIMEOUT with *code = code; with
 * arrive = 1 it stays 0.  Neither faults nor hangs the GPU.  limit_us in
 * [1, 1000000], code != 0, arrive in {0, 1}, else LLSA_ERR_ARG before any
 * launch. */
llsa_status llsa_selftest_wait_timeout(unsigned limit_us, int code, int arrive, llsa_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* LLSA_H */
