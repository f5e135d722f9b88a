// llsa_api.cu -- the C ABI: argument validation, buffer sizes, dispatch to the kernels.
#include <math.h>
#include <string.h>

#include <atomic>

#include "llsa_internal.cuh"

namespace llsa {

__device__ int g_device_error = 0;

static std::atomic<unsigned long long> g_launches{0};

void note_launches(int n) { g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed); }

int* device_error_word() {
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_device_error) != cudaSuccess) return nullptr;
  return (int*)ptr;
}

static int isqrt_exact(int B) {
  int t = 0;
  while ((t + 1) * (t + 1) <= B) ++t;
  return t * t == B ? t : -1;
}

llsa_status make_geo(const llsa_problem* p, Geo* g) {
  if (!p || !g) return LLSA_ERR_ARG;
  memset(g, 0, sizeof(*g));
  if (p->batch < 1 || p->heads < 1 || p->height < 1 || p->width < 1 || p->d < 1 || p->K < 1 || p->L < 1)
    return LLSA_ERR_ARG;
  if (p->dtype != LLSA_BF16 && p->dtype != LLSA_FP32) return LLSA_ERR_ARG;
  if (!(p->scale >= 0.0f) || isinf(p->scale)) return LLSA_ERR_ARG;
  if (p->L > LLSA_MAX_LEVELS) return LLSA_ERR_UNSUPPORTED;
  if (p->enrich_mask >> p->L) return LLSA_ERR_ARG;
  int t = isqrt_exact(p->B);
  if (t < 2) return LLSA_ERR_ARG;
  // block sizes whose queries map evenly onto a 128-thread block
  if (p->B != 4 && p->B != 16 && p->B != 64) return LLSA_ERR_UNSUPPORTED;
  if (p->d % 8 != 0 || p->d > 128) return LLSA_ERR_UNSUPPORTED;
  int64_t tl = 1;
  for (int l = 0; l < p->L; ++l) tl *= t;
  if (p->height % tl || p->width % tl) return LLSA_ERR_SHAPE;
  int64_t N = (int64_t)p->height * p->width;
  int64_t BH = (int64_t)p->batch * p->heads;
  if (N > (1ll << 30) || BH * N * p->d >= (1ll << 40) || BH > (1 << 24)) return LLSA_ERR_SHAPE;

  g->BH = (int)BH;
  g->H = p->height;
  g->W = p->width;
  g->N = (int)N;
  g->d = p->d;
  g->B = p->B;
  g->t = t;
  g->L = p->L;
  g->K = p->K;
  g->emask = p->enrich_mask;
  g->scale = p->scale > 0.0f ? p->scale : 1.0f / sqrtf((float)p->d);
  g->bf16 = p->dtype == LLSA_BF16;
  g->Bl[0] = 1;
  g->n[0] = (int)N;
  for (int l = 1; l <= p->L; ++l) {
    g->Bl[l] = g->Bl[l - 1] * p->B;
    g->n[l] = (int)(N / g->Bl[l]);
  }
  g->Kl[0] = 0;
  g->Kl[p->L] = g->n[p->L] < p->K ? g->n[p->L] : p->K;
  for (int l = p->L - 1; l >= 1; --l) {
    int64_t cand = (int64_t)g->Kl[l + 1] * p->B;
    g->Kl[l] = (int)(cand < p->K ? cand : p->K);
  }
  g->pyr_off[1] = g->idx_off[1] = g->offs_off[1] = g->cur_off[1] = 0;
  for (int l = 1; l <= p->L; ++l) {
    int64_t per = (int64_t)g->n[l] * g->Kl[l];
    if (per > INT32_MAX) return LLSA_ERR_SHAPE;   // CSC offsets are int32 per slice
    int64_t ncand = (l == p->L) ? g->n[l] : (int64_t)g->Kl[l + 1] * p->B;
    if (g->Kl[l] < ncand && ncand > kSelectMaxCandidates) return LLSA_ERR_UNSUPPORTED;
    g->pyr_off[l + 1] = g->pyr_off[l] + BH * g->n[l] * p->d;
    g->idx_off[l + 1] = g->idx_off[l] + BH * per;
    g->offs_off[l + 1] = g->offs_off[l] + BH * (g->n[l] + 1);
    g->cur_off[l + 1] = g->cur_off[l] + BH * g->n[l];
  }
  return LLSA_OK;
}

// Attention dispatch: bf16 problems with d = 64 and B = 16 run on the tensor
// cores; every other problem (fp32, other block sizes or head dims, K so large
// that a group's picks or pooled keys overflow the tiles) on the CUDA cores.
cudaError_t launch_attn_fwd(const Geo& g, const void* q, const void* k, const void* v, const float* pyrK,
                            const float* pyrV, const int32_t* idx, void* o, float* lse, cudaStream_t s) {
  if (attn_fwd_mma_supported(g)) return launch_attn_fwd_mma(g, q, k, v, pyrK, pyrV, idx, o, lse, s);
  return launch_attn_fwd_simt(g, q, k, v, pyrK, pyrV, idx, o, lse, s);
}

cudaError_t launch_attn_bwd(const Geo& g, const void* q, const void* k, const void* v, const void* o,
                            const void* dO, const float* lse, const float* pyrK, const float* pyrV,
                            const int32_t* idx, const int32_t* offs, const int32_t* qlist, void* dq, void* dk,
                            void* dv, void* workspace, cudaStream_t s) {
  if (attn_bwd_mma_supported(g))
    return launch_attn_bwd_mma(g, q, k, v, o, dO, lse, pyrK, pyrV, idx, offs, qlist, dq, dk, dv, workspace, s);
  return launch_attn_bwd_simt(g, q, k, v, o, dO, lse, pyrK, pyrV, idx, offs, qlist, dq, dk, dv, workspace, s);
}

}  // namespace llsa

using llsa::Geo;

static bool aligned16(const void* ptr) { return ptr && ((uintptr_t)ptr & 15u) == 0; }

static llsa_status launched(cudaError_t e) {
  if (e != cudaSuccess) return LLSA_ERR_CUDA;
  return cudaPeekAtLastError() == cudaSuccess ? LLSA_OK : LLSA_ERR_CUDA;
}

#define LLSA_GEO(p, g)                       \
  Geo g;                                     \
  do {                                       \
    llsa_status st_ = llsa::make_geo(p, &g); \
    if (st_ != LLSA_OK) return st_;          \
  } while (0)

#define LLSA_NEED(ptr)                       \
  do {                                       \
    if (!(ptr)) return LLSA_ERR_ARG;         \
    if (!aligned16(ptr)) return LLSA_ERR_ALIGN; \
  } while (0)

extern "C" {

const char* llsa_status_string(llsa_status s) {
  switch (s) {
    case LLSA_OK: return "ok";
    case LLSA_ERR_ARG: return "invalid argument";
    case LLSA_ERR_SHAPE: return "image does not tile into sqrt(B)^L squares, or sizes overflow";
    case LLSA_ERR_ALIGN: return "buffer not 16-byte aligned";
    case LLSA_ERR_WORKSPACE: return "workspace too small";
    case LLSA_ERR_CUDA: return "CUDA launch or runtime error";
    case LLSA_ERR_TIMEOUT: return "a bounded device-side wait gave up";
    case LLSA_ERR_UNSUPPORTED: return "problem outside what the kernels implement";
  }
  return "unknown status";
}

llsa_status llsa_validate(const llsa_problem* p) {
  LLSA_GEO(p, g);
  (void)g;
  return LLSA_OK;
}

llsa_status llsa_level_sizes(const llsa_problem* p, int64_t* n, int64_t* Kl) {
  if (!n || !Kl) return LLSA_ERR_ARG;
  LLSA_GEO(p, g);
  for (int l = 0; l <= g.L; ++l) {
    n[l] = g.n[l];
    Kl[l] = g.Kl[l];
  }
  return LLSA_OK;
}

llsa_status llsa_query_sizes(const llsa_problem* p, llsa_sizes* out) {
  if (!out) return LLSA_ERR_ARG;
  LLSA_GEO(p, g);
  size_t es = g.bf16 ? 2 : 4;
  out->tokens_bytes = (size_t)g.BH * g.N * g.d * es;
  out->lse_bytes = (size_t)g.BH * g.N * sizeof(float);
  out->pyramid_bytes = (size_t)g.pyr_off[g.L + 1] * sizeof(float);
  out->idx_bytes = (size_t)g.idx_off[g.L + 1] * sizeof(int32_t);
  out->offs_bytes = (size_t)g.offs_off[g.L + 1] * sizeof(int32_t);
  out->qlist_bytes = out->idx_bytes;
  size_t cur = ((size_t)g.cur_off[g.L + 1] * sizeof(int32_t) + 255) & ~(size_t)255;
  out->transpose_scratch_bytes = cur + out->idx_bytes;
  out->bwd_workspace_bytes = llsa::bwd_workspace_bytes(g);
  return LLSA_OK;
}

llsa_status llsa_reorder(const llsa_problem* p, const void* in, void* out, int to_hier, llsa_stream stream) {
  LLSA_GEO(p, g);
  LLSA_NEED(in);
  LLSA_NEED(out);
  size_t bytes = (size_t)g.BH * g.N * g.d * (g.bf16 ? 2 : 4);
  const char* a = (const char*)in;
  const char* b = (const char*)out;
  if (a < b + bytes && b < a + bytes) return LLSA_ERR_ARG;   // must not overlap
  return launched(llsa::launch_reorder(g, in, out, to_hier, (cudaStream_t)stream));
}

llsa_status llsa_pool(const llsa_problem* p, const void* x, float* pyramid, llsa_stream stream) {
  LLSA_GEO(p, g);
  LLSA_NEED(x);
  LLSA_NEED(pyramid);
  return launched(llsa::launch_pool(g, x, pyramid, (cudaStream_t)stream));
}

llsa_status llsa_select_level(const llsa_problem* p, int level, const float* pyrQ, const float* pyrK,
                              int32_t* idx, llsa_stream stream) {
  LLSA_GEO(p, g);
  if (level < 1 || level > g.L) return LLSA_ERR_ARG;
  LLSA_NEED(pyrQ);
  LLSA_NEED(pyrK);
  LLSA_NEED(idx);
  return launched(llsa::launch_select_level(g, level, pyrQ, pyrK, idx, (cudaStream_t)stream));
}

llsa_status llsa_select(const llsa_problem* p, const float* pyrQ, const float* pyrK, int32_t* idx,
                        llsa_stream stream) {
  LLSA_GEO(p, g);
  LLSA_NEED(pyrQ);
  LLSA_NEED(pyrK);
  LLSA_NEED(idx);
  for (int l = g.L; l >= 1; --l) {
    llsa_status st = launched(llsa::launch_select_level(g, l, pyrQ, pyrK, idx, (cudaStream_t)stream));
    if (st != LLSA_OK) return st;
  }
  return LLSA_OK;
}

llsa_status llsa_attn_fwd(const llsa_problem* p, const void* q, const void* k, const void* v,
                          const float* pyrK, const float* pyrV, const int32_t* idx, void* o, float* lse,
                          llsa_stream stream) {
  LLSA_GEO(p, g);
  LLSA_NEED(q);
  LLSA_NEED(k);
  LLSA_NEED(v);
  LLSA_NEED(pyrK);
  LLSA_NEED(pyrV);
  LLSA_NEED(idx);
  LLSA_NEED(o);
  LLSA_NEED(lse);
  return launched(llsa::launch_attn_fwd(g, q, k, v, pyrK, pyrV, idx, o, lse, (cudaStream_t)stream));
}

llsa_status llsa_index_transpose(const llsa_problem* p, const int32_t* idx, int32_t* offs, int32_t* qlist,
                                 void* scratch, llsa_stream stream) {
  LLSA_GEO(p, g);
  LLSA_NEED(idx);
  LLSA_NEED(offs);
  LLSA_NEED(qlist);
  LLSA_NEED(scratch);
  return launched(llsa::launch_index_transpose(g, idx, offs, qlist, (int32_t*)scratch, (cudaStream_t)stream));
}

llsa_status llsa_attn_bwd(const llsa_problem* p, const void* q, const void* k, const void* v,
                          const void* o, const void* dO, const float* lse, const float* pyrK,
                          const float* pyrV, const int32_t* idx, const int32_t* offs, const int32_t* qlist,
                          void* dq, void* dk, void* dv, void* workspace, llsa_stream stream) {
  LLSA_GEO(p, g);
  LLSA_NEED(q);
  LLSA_NEED(k);
  LLSA_NEED(v);
  LLSA_NEED(o);
  LLSA_NEED(dO);
  LLSA_NEED(lse);
  LLSA_NEED(pyrK);
  LLSA_NEED(pyrV);
  LLSA_NEED(idx);
  LLSA_NEED(offs);
  LLSA_NEED(qlist);
  LLSA_NEED(dq);
  LLSA_NEED(dk);
  LLSA_NEED(dv);
  LLSA_NEED(workspace);
  return launched(llsa::launch_attn_bwd(g, q, k, v, o, dO, lse, pyrK, pyrV, idx, offs, qlist, dq, dk, dv,
                                        workspace, (cudaStream_t)stream));
}

llsa_status llsa_attn_paths(const llsa_problem* p, int* fwd_tc, int* bwd_tc) {
  LLSA_GEO(p, g);
  if (fwd_tc) *fwd_tc = llsa::attn_fwd_mma_supported(g) ? 1 : 0;
  if (bwd_tc) *bwd_tc = llsa::attn_bwd_mma_supported(g) ? 1 : 0;
  return LLSA_OK;
}

uint64_t llsa_kernel_launches(void) { return (uint64_t)llsa::g_launches.load(std::memory_order_relaxed); }

llsa_status llsa_device_error(llsa_stream stream, int* code) {
  if (!code) return LLSA_ERR_ARG;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return LLSA_ERR_CUDA;
  int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, llsa::g_device_error, sizeof(int)) != cudaSuccess) return LLSA_ERR_CUDA;
  if (cudaMemcpyToSymbol(llsa::g_device_error, &zero, sizeof(int)) != cudaSuccess) return LLSA_ERR_CUDA;
  *code = v;
  return v ? LLSA_ERR_TIMEOUT : LLSA_OK;
}

}  // extern "C"
