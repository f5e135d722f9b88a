// llsa_internal.cuh -- shared definitions of the CUDA side (never seen by callers).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "llsa.h"

namespace llsa {

// Derived sizes of one problem, computed on the host and passed to kernels by value.
struct Geo {
  int BH;          // batch * heads
  int H, W;        // image size
  int N;           // tokens per slice
  int d;           // head dimension
  int B;           // block size
  int t;           // sqrt(B)
  int L;           // levels
  int K;           // requested top-K
  unsigned emask;  // enriched levels, bit l-1 = level l
  float scale;     // softmax scale
  int bf16;        // 1: bf16 tensors, 0: fp32
  int n[LLSA_MAX_LEVELS + 1];        // tokens per level (n[0] = N)
  int Kl[LLSA_MAX_LEVELS + 1];       // list length per level (Kl[0] = 0)
  int64_t Bl[LLSA_MAX_LEVELS + 1];   // B^l
  int64_t pyr_off[LLSA_MAX_LEVELS + 2];   // element offset of level l in a pyramid (index L+1 = total)
  int64_t idx_off[LLSA_MAX_LEVELS + 2];   // element offset of level l in idx / qlist
  int64_t offs_off[LLSA_MAX_LEVELS + 2];  // element offset of level l in offs
  int64_t cur_off[LLSA_MAX_LEVELS + 2];   // element offset of level l in the transpose cursors
};

// Fills g from p; returns LLSA_OK or the validation error.
llsa_status make_geo(const llsa_problem* p, Geo* g);

// Counts kernel launches issued by this library (host side, process wide).
void note_launches(int n);

// Device address of the error word that bounded waits set when they give up
// (nullptr if the symbol cannot be resolved on the current device).
int* device_error_word();

// ----------------------------------------------------------------- launchers
// All return cudaSuccess or the launch error; they assume a validated Geo.
cudaError_t launch_reorder(const Geo& g, const void* in, void* out, int to_hier, cudaStream_t s);
cudaError_t launch_pool(const Geo& g, const void* x, float* pyr, cudaStream_t s);
cudaError_t launch_select_level(const Geo& g, int level, const float* pyrQ, const float* pyrK, int32_t* idx,
                                cudaStream_t s);
cudaError_t launch_index_transpose(const Geo& g, const int32_t* idx, int32_t* offs, int32_t* qlist,
                                   int32_t* cursor, cudaStream_t s);
cudaError_t launch_attn_fwd(const Geo& g, const void* q, const void* k, const void* v, const float* pyrK,
                            const float* pyrV, const int32_t* idx, void* o, float* lse, cudaStream_t s);
cudaError_t launch_attn_bwd(const Geo& g, const void* q, const void* k, const void* v, const void* o,
                            const void* dO, const float* lse, const float* pyrK, const float* pyrV,
                            const int32_t* idx, const int32_t* offs, const int32_t* qlist, void* dq, void* dk,
                            void* dv, void* workspace, cudaStream_t s);

// CUDA-core (fp32 FMA) attention kernels.
cudaError_t launch_attn_fwd_simt(const Geo& g, const void* q, const void* k, const void* v, const float* pyrK,
                                 const float* pyrV, const int32_t* idx, void* o, float* lse, cudaStream_t s);
cudaError_t launch_attn_bwd_simt(const Geo& g, const void* q, const void* k, const void* v, const void* o,
                                 const void* dO, const float* lse, const float* pyrK, const float* pyrV,
                                 const int32_t* idx, const int32_t* offs, const int32_t* qlist, void* dq, void* dk,
                                 void* dv, void* workspace, cudaStream_t s);

struct BwdWorkspace;

// Tensor maps of one token tensor whose boxes carry 1..kRunMax blocks of 16
// rows (a run of consecutive blocks is then one TMA copy: issuing a copy
// costs about as much as moving a 2 KB tile).
constexpr int kRunMax = 4;
struct RunMaps {
  CUtensorMap m[kRunMax];
};
cudaError_t make_run_maps(RunMaps* maps, const void* base, int64_t rows);

// Tensor-core attention kernels (bf16, d = 64, B = 16).
bool attn_bwd_mma_supported(const Geo& g);
cudaError_t launch_attn_bwd_mma(const Geo& g, const void* q, const void* k, const void* v, const void* o,
                                const void* dO, const float* lse, const float* pyrK, const float* pyrV,
                                const int32_t* idx, const int32_t* offs, const int32_t* qlist, void* dq, void* dk,
                                void* dv, void* workspace, cudaStream_t s);
// Query-major backward on tcgen05: dQ, D = rowsum(dO * O), and the pooled
// gradients of levels >= 2 (atomics into ws.dPK / ws.dPV, zeroed by the caller).
cudaError_t launch_attn_bwd_q_tc(const Geo& g, const void* q, const void* k, const void* v, const void* o,
                                 const void* dO, const float* lse, const float* pyrK, const float* pyrV,
                                 const int32_t* idx, const int32_t* offs, const int32_t* qlist,
                                 const BwdWorkspace& ws, void* dq, cudaStream_t s);
cudaError_t launch_attn_bwd_kv_tc(const Geo& g, const void* k, const void* v, const RunMaps& tq,
                                  const RunMaps& tdo, const float* lse, const int32_t* offs,
                                  const BwdWorkspace& ws, void* dk, void* dv, cudaStream_t s);
bool attn_fwd_mma_supported(const Geo& g);
cudaError_t launch_attn_fwd_mma(const Geo& g, const void* q, const void* k, const void* v, const float* pyrK,
                                const float* pyrV, const int32_t* idx, void* o, float* lse, cudaStream_t s);

// TMA descriptor of a [rows][64] bf16 token tensor with boxes of `box_rows`
// rows (1..256) x 64 columns (16 rows: one 2 KB key or query block),
// 128-byte swizzle.
cudaError_t make_token_map_box(CUtensorMap* map, const void* base, int64_t rows, int box_rows);

// Largest candidate count the selection kernel keeps in shared memory.
constexpr int kSelectMaxCandidates = 24576;   // 192 KB of 64-bit keys, one warp

// Workspace of the backward pass: D [BH][N] fp32, the fp32 level gradients
// of the pooled K and of the pooled V (each a pyramid), two work counters
// (key groups claimed by the key-major pass, tokens by the query-major pass), then
// the query groups' unions (each entry block << 8 | pick mask, laid out like
// the level-1 index lists) and their sizes, one tile of the pooled keys of
// levels >= 2 per level-2 token (kBwdCoarseTileBytes each), then the key
// groups' unions (laid out like the level-1 CSC lists) and their sizes.
struct BwdWorkspace {
  float* D;
  float* dPK;
  float* dPV;
  int* counter;
  int32_t* ulist;
  int32_t* ucount;
  unsigned char* ctile;
  int32_t* ulist_kv;
  int32_t* ucount_kv;
  size_t zero_bytes;   // bytes from dPK on that must start at zero (sums and counters)
};

// A level-2 token's pooled keys of levels >= 2 (at most 32): K and V rows as
// bf16 [32][64] with the 128-byte swizzle, then per row the logit bias
// (log2 domain; -inf: no key), the level and the pooled token id (-1: none).
constexpr size_t kBwdCoarseTileBytes = 2 * 32 * 128 + 3 * 32 * 4;

inline size_t bwd_round256(size_t x) { return (x + 255) & ~(size_t)255; }

inline size_t bwd_pyr_bytes(const Geo& g) { return bwd_round256((size_t)g.pyr_off[g.L + 1] * sizeof(float)); }

inline size_t bwd_workspace_bytes(const Geo& g) {
  const size_t dsz = bwd_round256((size_t)g.BH * g.N * sizeof(float));
  const size_t usz = bwd_round256((size_t)g.BH * g.n[1] * g.Kl[1] * sizeof(int32_t));
  const size_t csz = bwd_round256(((size_t)g.BH * g.n[1] / 8 + 1) * sizeof(int32_t));
  const size_t tsz = bwd_round256(((size_t)g.BH * g.n[1] / 16 + 1) * kBwdCoarseTileBytes);
  return dsz + 2 * bwd_pyr_bytes(g) + 256 + 2 * (usz + csz) + tsz;
}

inline BwdWorkspace carve_bwd_workspace(const Geo& g, void* workspace) {
  const size_t dsz = bwd_round256((size_t)g.BH * g.N * sizeof(float));
  const size_t pyr = bwd_pyr_bytes(g);
  const size_t usz = bwd_round256((size_t)g.BH * g.n[1] * g.Kl[1] * sizeof(int32_t));
  const size_t csz = bwd_round256(((size_t)g.BH * g.n[1] / 8 + 1) * sizeof(int32_t));
  const size_t tsz = bwd_round256(((size_t)g.BH * g.n[1] / 16 + 1) * kBwdCoarseTileBytes);
  char* b = static_cast<char*>(workspace);
  char* after = b + dsz + 2 * pyr + 256;
  char* kv = after + usz + csz + tsz;
  return BwdWorkspace{reinterpret_cast<float*>(b),
                      reinterpret_cast<float*>(b + dsz),
                      reinterpret_cast<float*>(b + dsz + pyr),
                      reinterpret_cast<int*>(b + dsz + 2 * pyr),
                      reinterpret_cast<int32_t*>(after),
                      reinterpret_cast<int32_t*>(after + usz),
                      reinterpret_cast<unsigned char*>(after + usz + csz),
                      reinterpret_cast<int32_t*>(kv),
                      reinterpret_cast<int32_t*>(kv + usz),
                      2 * pyr + 2 * sizeof(int)};
}

// ------------------------------------------------------------ device helpers

// TMA boxes over a chunk's blocks: lane j < nq holds block id b (ascending
// over the lanes).  Returns how many blocks (1..kRunMax) the box starting at
// block j carries -- runs of consecutive ids share a box -- or 0 when block j
// lies inside an earlier lane's box.  Every lane of the warp calls it.
__device__ __forceinline__ int run_box(int b, int nq, int lane) {
  const int prev = __shfl_up_sync(0xffffffffu, b, 1);
  const bool brk = lane == 0 || b != prev + 1;
  const unsigned starts = __ballot_sync(0xffffffffu, lane < nq && brk);
  if (lane >= nq) return 0;
  const int rs = 31 - __clz(starts & ((2u << lane) - 1u));    // start of the run
  if ((lane - rs) % kRunMax) return 0;
  const unsigned later = starts & ~((2u << lane) - 1u);
  const int rend = later ? __ffs(later) - 1 : nq;              // end of the run
  return min(kRunMax, rend - lane);
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

}  // namespace llsa
