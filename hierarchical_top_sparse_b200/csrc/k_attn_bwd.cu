// k_attn_bwd.cu -- the tensor-core sparse attention backward (bf16, d = 64,
// B = 16) in two passes on tcgen05 (Trainable Log-linear Sparse Attention
// summary §4.1, "trainable" in its title):
//
//  * query-major pass (k_attn_bwd_q_tc.cu), per level-2 token (two groups of
//    8 query blocks): D = rowsum(dO * O); S and dP against the union of the
//    groups' picked key blocks and against the token's pooled keys of levels
//    >= 2; dS = P (dP - D); dQ = scale * dS K; the pooled keys' gradients
//    scale * dS^T Q and P^T dO summed over the token in tensor memory, then
//    one fp32 atomic per (pooled token, channel).
//  * key-major pass (k_attn_bwd_kv_tc.cu), per group of 8 fine key blocks,
//    over the union of their level-1 CSC query lists: dV, dK, and the
//    pooled-key gradients of levels >= 2 spread back over the B^l tokens
//    they average.
//
// A level-1 pooled token is the mean of the 16 keys of the block it stands
// for, and the queries that attend it are exactly those that picked that
// block.  So level-1 enrichment folds into both passes with no extra loads:
// its logit is the mean of the block's 16 fine logits plus ln B, its dP is the
// mean of the 16 fine dP, and its P and dS add P_c / B and dS_c / B to each of
// the block's 16 fine entries (hierarchical KV enrichment, §四).
#include "llsa_internal.cuh"

namespace llsa {

constexpr int kBwdCoarseMax = 32;   // pooled keys of levels >= 2 per query block that the passes hold
// Largest level-1 list the tensor-core passes take: the K = all lists of a
// 256 x 256 image (every one of its 4096 blocks), the largest case the GPU
// tests run them on.  Longer lists go to the CUDA-core kernels.
constexpr int kBwdMaxK1 = 4096;

bool attn_bwd_mma_supported(const Geo& g) {
  if (!g.bf16 || g.d != 64 || g.B != 16) return false;
  if (g.n[1] % 16) return false;    // whole level-2 tokens: two groups of 8 query blocks
  if (g.n[1] >= (1 << 23)) return false;   // union entries pack (block << 8) | mask into 32 bits
  if (g.Kl[1] < 1 || g.Kl[1] > kBwdMaxK1) return false;
  int nc = 0;
  for (int l = 2; l <= g.L; ++l)
    if ((g.emask >> (l - 1)) & 1u) nc += g.Kl[l];
  if (nc > kBwdCoarseMax) return false;
  if ((int64_t)g.BH * g.N >= (1ll << 31)) return false;
  if ((int64_t)g.BH * g.n[1] * g.Kl[1] >= (1ll << 31)) return false;
  return true;
}

cudaError_t launch_attn_bwd_mma(const Geo& g, const void* q, const void* k, const void* v, const void* o,
                                const void* dO, const float* lse, const float* pyrK, const float* pyrV,
                                const int32_t* idx, const int32_t* offs, const int32_t* qlist, void* dq, void* dk,
                                void* dv, void* workspace, cudaStream_t s) {
  const int64_t rows = (int64_t)g.BH * g.N;
  RunMaps tq, tdo;   // boxes of 1..4 query blocks: the key-major pass stacks them
  cudaError_t e = make_run_maps(&tq, q, rows);
  if (e == cudaSuccess) e = make_run_maps(&tdo, dO, rows);
  if (e != cudaSuccess) return e;
  BwdWorkspace ws = carve_bwd_workspace(g, workspace);
  e = cudaMemsetAsync(ws.dPK, 0, ws.zero_bytes, s);   // pooled-key sums and the work counter
  if (e != cudaSuccess) return e;
  e = launch_attn_bwd_q_tc(g, q, k, v, o, dO, lse, pyrK, pyrV, idx, offs, qlist, ws, dq, s);
  if (e != cudaSuccess) return e;
  return launch_attn_bwd_kv_tc(g, k, v, tq, tdo, lse, offs, ws, dk, dv, s);
}

}  // namespace llsa
