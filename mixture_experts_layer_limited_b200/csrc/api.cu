// C-ABI entry points of libmoe (declared in include/moe.h): argument checks on
// the host, TMA tensor-map encoding, kernel launches. No allocation happens
// here; every buffer belongs to the caller.
#include <atomic>
#include <mutex>

#include "kernels.cuh"


using namespace moe;

namespace {

thread_local int32_t g_last_cuda_error = 0;

moe_status cuda_fail(int32_t code) {
  g_last_cuda_error = code;
  return MOE_ERR_CUDA;
}

moe_status check_launch(cudaError_t e) {
  if (e != cudaSuccess) return cuda_fail(static_cast<int32_t>(e));
  return MOE_OK;
}

bool misaligned(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }

template <typename... P>
bool any_misaligned(P... ps) {
  return (misaligned(ps) || ...);
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, looked up once through the runtime (so the
// library needs no link-time dependency on libcuda).
EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Row-major [outer, inner] matrix; box = 128 bytes of `inner` x box_rows rows,
// 128-byte swizzle (the layout the tcgen05 smem descriptors expect).
moe_status make_tmap(CUtensorMap* m, const void* ptr, bool one_byte, uint64_t inner, uint64_t outer,
                     uint32_t box_rows) {
  EncodeTiledFn enc = encode_tiled();
  if (!enc) return cuda_fail(static_cast<int32_t>(cudaErrorNotSupported));
  const uint64_t esize = one_byte ? 1 : 2;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * esize};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / esize), box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, one_byte ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                   const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cuda_fail(1000 + static_cast<int32_t>(r));
  return MOE_OK;
}

// Token-row maps of a grouped GEMM: bf16 rows are fetched with 256-, 128-,
// 64-, 32- and 16-row boxes; e4m3 rows (at most 32 tokens a tile) with one
// 32-row box.
moe_status make_token_tmaps(TokenMaps* m, const void* ptr, bool fp8, uint64_t K, uint64_t rows) {
  if (fp8) return make_tmap(&m->box[0], ptr, true, K, rows, 32);
  for (int i = 0; i < kTokBoxes; ++i) {
    moe_status s = make_tmap(&m->box[i], ptr, false, K, rows, 256u >> i);
    if (s != MOE_OK) return s;
  }
  return MOE_OK;
}

moe_status sm_count(int* n) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  e = cudaDeviceGetAttribute(n, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(e);
  return MOE_OK;
}

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// Limit of every bounded device-side wait, passed to the kernels at launch
// (moe_set_wait_limit_ns; 2 s unless changed).
std::atomic<uint64_t> g_wait_limit_ns{kDefaultWaitLimitNs};
uint64_t wait_limit() { return g_wait_limit_ns.load(std::memory_order_relaxed); }

}  // namespace

extern "C" {

int32_t moe_abi_version(void) { return MOE_ABI_VERSION; }

int32_t moe_last_cuda_error(void) { return g_last_cuda_error; }

moe_status moe_set_wait_limit_ns(uint64_t ns) {
  g_wait_limit_ns.store(ns == 0 ? kDefaultWaitLimitNs : ns, std::memory_order_relaxed);
  return MOE_OK;
}

uint64_t moe_wait_limit_ns(void) { return wait_limit(); }

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case MOE_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_DEVICE_CHECK: return "device-side bounds check failed";
    case MOE_ERR_DEVICE_TIMEOUT: return "device-side bounded wait timed out";
    default: return "unknown status";
  }
}

// logits = x @ gate^T on the clustered gate GEMM (r carries T, H, E, logits,
// status), and with `route` the routing of every token in the same launch
moe_status gate_gemm(const RouteArgs& r, const void* x, const void* gate_w, bool route, int nsm, cudaStream_t st) {
  CUtensorMap tmX, tmG;
  moe_status s = make_tmap(&tmX, x, false, r.H, r.T, 128);
  if (s != MOE_OK) return s;
  s = make_tmap(&tmG, gate_w, false, r.H, r.E, static_cast<uint32_t>(r.E));
  if (s != MOE_OK) return s;
  return check_launch(launch_gate_gemm(tmX, tmG, r, route, nsm, st));
}

moe_status moe_gate_logits(int32_t T, int32_t H, int32_t E, const void* x, const void* gate_w, float* logits,
                           int32_t* dev_status, void* stream) {
  if (T < 1 || H < 64 || !x || !gate_w || !logits) return MOE_ERR_INVALID_ARG;
  if (H % 64 != 0 || E > 256 || E < 16 || E % 16 != 0) return MOE_ERR_UNSUPPORTED;
  if (any_misaligned(x, gate_w, logits)) return MOE_ERR_ALIGNMENT;
  int nsm = 0;
  moe_status s = sm_count(&nsm);
  if (s != MOE_OK) return s;
  RouteArgs r{};
  r.T = T;
  r.H = H;
  r.E = E;
  r.logits = logits;
  r.status = dev_status;
  r.wait_ns = wait_limit();
  return gate_gemm(r, x, gate_w, false, nsm, as_stream(stream));
}

moe_status moe_route(const moe_route_params* p, const void* x, const void* gate_w, const float* sel_bias,
                     float* logits, int32_t* topk_ids, float* topk_w, int32_t* expert_counts, void* stream) {
  if (!p || !topk_ids || !topk_w || !expert_counts || !logits) return MOE_ERR_INVALID_ARG;
  if (p->T < 1 || p->k < 1 || p->n_group < 1 || p->topk_group < 1) return MOE_ERR_INVALID_ARG;
  if (p->scoring != MOE_SOFTMAX && p->scoring != MOE_SIGMOID) return MOE_ERR_INVALID_ARG;
  if (p->E < 1 || p->E % p->n_group != 0 || p->topk_group > p->n_group) return MOE_ERR_INVALID_ARG;
  if (p->k > p->topk_group * (p->E / p->n_group)) return MOE_ERR_INVALID_ARG;
  if (p->k > 16 || p->E > 256 || p->E < 16 || p->E % 16 != 0 || p->n_group > 32) return MOE_ERR_UNSUPPORTED;
  if (x) {
    if (!gate_w || p->H < 64) return MOE_ERR_INVALID_ARG;
    if (p->H % 64 != 0) return MOE_ERR_UNSUPPORTED;
  }
  if (any_misaligned(x, gate_w, sel_bias, logits, topk_ids, topk_w, expert_counts)) return MOE_ERR_ALIGNMENT;
  int nsm = 0;
  moe_status s = sm_count(&nsm);
  if (s != MOE_OK) return s;
  cudaStream_t st = as_stream(stream);
  RouteArgs r{p->T, p->H, p->E, p->k, p->n_group, p->topk_group, p->scoring, p->norm_topk_prob ? 1 : 0,
              p->routed_scaling_factor, sel_bias, logits, topk_ids, topk_w, expert_counts, p->dev_status,
              wait_limit()};
  cudaError_t e = cudaMemsetAsync(expert_counts, 0, sizeof(int32_t) * p->E, st);
  if (e != cudaSuccess) return cuda_fail(e);
  // from x: one launch (projection + routing) where the shape allows
  if (x) {
    const bool fused = route8_experts_per_thread(r) > 0;
    if ((s = gate_gemm(r, x, gate_w, fused, nsm, st)) != MOE_OK) return s;
    if (fused) return MOE_OK;
  }
  return check_launch(launch_route_tokens(r, nsm, st));
}

moe_status moe_permute_workspace_size(int32_t T, int32_t k, int32_t E, size_t* bytes) {
  if (!bytes || T < 1 || k < 1 || E < 1) return MOE_ERR_INVALID_ARG;
  *bytes = permute_workspace_bytes(T, E);
  return MOE_OK;
}

moe_status moe_permute(int32_t T, int32_t k, int32_t E, int32_t H, const int32_t* topk_ids,
                       const float* topk_w, const void* x, moe_dtype x_dtype, const float* x_scale,
                       void* x_perm, moe_dtype perm_dtype, float* x_perm_scale, void* x_q, float* x_q_scale,
                       int32_t* expert_offsets, int32_t* src_token, int32_t* slot_to_row, float* row_w,
                       void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream) {
  if (T < 1 || k < 1 || E < 1 || H < 1 || k > E) return MOE_ERR_INVALID_ARG;
  if (!topk_ids || !expert_offsets || !src_token || !slot_to_row || !workspace) return MOE_ERR_INVALID_ARG;
  if (row_w && !topk_w) return MOE_ERR_INVALID_ARG;
  if ((x_perm || x_q) && !x) return MOE_ERR_INVALID_ARG;
  if (x_dtype != MOE_BF16 && x_dtype != MOE_E4M3) return MOE_ERR_INVALID_ARG;
  if (perm_dtype != MOE_BF16 && perm_dtype != MOE_E4M3) return MOE_ERR_INVALID_ARG;
  if (x_dtype == MOE_E4M3 && perm_dtype != MOE_E4M3) return MOE_ERR_UNSUPPORTED;
  const bool quant = x_dtype == MOE_BF16 && perm_dtype == MOE_E4M3;
  if ((x_q || x_q_scale) && (!quant || !x_q || !x_q_scale)) return MOE_ERR_INVALID_ARG;
  if (k > 16 || E > 1024) return MOE_ERR_UNSUPPORTED;
  if (static_cast<long long>(T) * k > 0x7fffffffLL) return MOE_ERR_UNSUPPORTED;
  if (perm_dtype == MOE_BF16) {
    if (H % 8 != 0) return MOE_ERR_UNSUPPORTED;
  } else {
    if (H % 128 != 0) return MOE_ERR_UNSUPPORTED;
    if (x_perm && !x_perm_scale) return MOE_ERR_INVALID_ARG;
    if (x_dtype == MOE_E4M3 && x_perm && !x_scale) return MOE_ERR_INVALID_ARG;
  }
  if (workspace_bytes < permute_workspace_bytes(T, E)) return MOE_ERR_INVALID_ARG;
  if (any_misaligned(topk_ids, topk_w, x, x_scale, x_perm, x_perm_scale, x_q, x_q_scale, expert_offsets,
                     src_token, slot_to_row, row_w, workspace))
    return MOE_ERR_ALIGNMENT;
  return check_launch(launch_permute(T, k, E, H, x_dtype == MOE_E4M3, perm_dtype == MOE_E4M3, topk_ids, topk_w, x,
                                     x_scale, x_perm, x_perm_scale, x_q, x_q_scale, expert_offsets, src_token,
                                     slot_to_row, row_w, static_cast<int32_t*>(workspace), dev_status,
                                     as_stream(stream)));
}

}  // extern "C"

namespace {

// Shared checks of the grouped SwiGLU calls; `a` is the GEMM's activation
// operand (x for the first GEMM, h for the second).
moe_status check_ffn(int32_t rows, int32_t H, const moe_ffn_weights* w, const void* a,
                     const float* a_scale, bool need_w13, bool need_w2) {
  if (!w || !a) return MOE_ERR_INVALID_ARG;
  if ((need_w13 && !w->w13) || (need_w2 && !w->w2)) return MOE_ERR_INVALID_ARG;
  if (rows < 1 || H < 1 || w->I < 1 || w->groups < 1) return MOE_ERR_INVALID_ARG;
  if (w->dtype != MOE_BF16 && w->dtype != MOE_E4M3) return MOE_ERR_INVALID_ARG;
  if (w->tiled != 0 && w->tiled != 1) return MOE_ERR_INVALID_ARG;
  if (w->tiled && w->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (H % 256 != 0 || w->I % 128 != 0 || w->groups > 512) return MOE_ERR_UNSUPPORTED;
  if (w->dtype == MOE_E4M3) {
    if ((need_w13 && !w->w13_scale) || (need_w2 && !w->w2_scale) || !a_scale) return MOE_ERR_INVALID_ARG;
    if (H > 8192 || w->I > 8192) return MOE_ERR_UNSUPPORTED;
  }
  if (static_cast<long long>(w->groups) * 2 * w->I > 0x7fffffffLL ||
      static_cast<long long>(w->groups) * H > 0x7fffffffLL)
    return MOE_ERR_UNSUPPORTED;
  // the tiled view's rows are TMA coordinates (int32)
  if (w->tiled && static_cast<long long>(w->groups) * 2 * w->I * (H / 64) > 0x7fffffffLL) return MOE_ERR_UNSUPPORTED;
  if (any_misaligned(w->w13, w->w2, w->w13_scale, w->w2_scale, a, a_scale)) return MOE_ERR_ALIGNMENT;
  return MOE_OK;
}

// Token blocks (of at most 256 rows) of `rows` rows in one segment, and an
// upper bound over `groups` segments of `rows` rows in all (each non-empty
// segment adds at most one partial block).
int32_t ffn_blocks(int32_t rows) { return (rows + 255) / 256; }
int32_t ffn_routed_blocks(int32_t rows, int32_t groups) { return ffn_blocks(rows) + groups; }

// Tensor maps and kernel arguments of one grouped GEMM.
struct GemmPlan {
  CUtensorMap tmA;
  TokenMaps tmB;
  GemmArgs g;
  bool fp8;
};

// Kernel choice for the bf16 grouped GEMMs, by measurement at the V3 shape on
// B200: single CTAs, 256-token tiles with one TMEM accumulator pair, three
// 64-K stages; 4 epilogue warps for gate/up and 12 for down, whose output
// rows are twice as wide (three warps per TMEM lane quarter take turns on
// its 32-token chunks). E4M3: at most 32 tokens a tile.
moe_status plan_gate_up(int32_t rows, int32_t H, const moe_ffn_weights* w, const void* a, const float* a_scale,
                        const int32_t* offsets, void* h_ws, float* h_scale_ws, int32_t* dev_status, GemmPlan* p) {
  const bool fp8 = w->dtype == MOE_E4M3;
  const int I = w->I;
  // tiled weights: a [*, 64] matrix whose 256-row boxes (128 gate rows, then
  // the same features' 128 up rows) are the tiles
  moe_status s = w->tiled ? make_tmap(&p->tmA, w->w13, false, 64, static_cast<uint64_t>(w->groups) * 2 * I * (H / 64), 256)
                          : make_tmap(&p->tmA, w->w13, fp8, H, static_cast<uint64_t>(w->groups) * 2 * I, 128);
  if (s != MOE_OK) return s;
  if ((s = make_token_tmaps(&p->tmB, a, fp8, H, rows)) != MOE_OK) return s;
  GemmArgs& g = p->g;
  g = GemmArgs{};
  g.rows = rows;
  g.K = H;
  g.groups = w->groups;
  g.offsets = offsets;
  g.a_rows_per_group = 2 * I;            // w13[e]: gate rows [0, I), up rows [I, 2I)
  g.a_tiled = w->tiled;
  g.n_mblk = I / 128;
  g.mblk_stride = 128;
  g.sub1_off = I;                        // sub-tile 1: the up rows of the same 128 features
  g.feat_stride = 128;
  g.bn_max = fp8 ? 32 : 256;
  g.out = h_ws;
  g.out_ld = I;
  g.a_scale = w->w13_scale;
  g.b_scale = a_scale;
  g.out_scale = h_scale_ws;
  g.status = dev_status;
  g.epi_warps = 4;
  g.wait_ns = wait_limit();
  p->fp8 = fp8;
  return MOE_OK;
}

moe_status plan_down(int32_t rows, int32_t H, const moe_ffn_weights* w, const void* h, const float* h_scale,
                     const int32_t* offsets, const float* row_w, void* out, int32_t* dev_status, GemmPlan* p) {
  const bool fp8 = w->dtype == MOE_E4M3;
  const int I = w->I;
  // bf16: a tile's 256 contiguous w2 rows are one TMA box
  moe_status s = w->tiled ? make_tmap(&p->tmA, w->w2, false, 64, static_cast<uint64_t>(w->groups) * H * (I / 64), 256)
                          : make_tmap(&p->tmA, w->w2, fp8, I, static_cast<uint64_t>(w->groups) * H, fp8 ? 128 : 256);
  if (s != MOE_OK) return s;
  if ((s = make_token_tmaps(&p->tmB, h, fp8, I, rows)) != MOE_OK) return s;
  GemmArgs& g = p->g;
  g = GemmArgs{};
  g.rows = rows;
  g.K = I;
  g.groups = w->groups;
  g.offsets = offsets;
  g.a_rows_per_group = H;
  g.a_tiled = w->tiled;
  g.n_mblk = H / 256;
  g.mblk_stride = 256;
  g.sub1_off = 128;                      // sub-tiles: w2 rows [mb*256, +128) and [mb*256 + 128, +128)
  g.feat_stride = 256;
  g.feat_sub1 = 128;
  g.bn_max = fp8 ? 32 : 256;
  g.a_one_box = fp8 ? 0 : 1;
  g.out = out;
  g.out_ld = H;
  g.row_w = row_w;
  g.a_scale = w->w2_scale;
  g.b_scale = h_scale;
  g.status = dev_status;
  g.epi_warps = 12;
  g.wait_ns = wait_limit();
  p->fp8 = fp8;
  return MOE_OK;
}

moe_status launch_plan(const GemmPlan& p, int epi, cudaStream_t st, int nsm, const GemmPlan* second = nullptr) {

  // one launch needs the same kernel form for both: bf16, same tile shape
  const bool one = second && !p.fp8 && !second->fp8 && p.g.bn_max == second->g.bn_max &&
                   p.g.epi_warps == second->g.epi_warps;
  if (second && !one) {
    moe_status s = check_launch(launch_grouped_gemm(p.fp8, epi, p.tmA, p.tmB, p.g, nsm, st));
    return s != MOE_OK ? s : check_launch(launch_grouped_gemm(second->fp8, epi, second->tmA, second->tmB,
                                                              second->g, nsm, st));
  }
  if (!second) return check_launch(launch_grouped_gemm(p.fp8, epi, p.tmA, p.tmB, p.g, nsm, st));
  const SecondProblem two{second->tmA, second->tmB, second->g};
  return check_launch(launch_grouped_gemm(p.fp8, epi, p.tmA, p.tmB, p.g, nsm, st, &two));
}

moe_status run_gate_up(int32_t rows, int32_t H, const moe_ffn_weights* w, const void* a,
                       const float* a_scale, const int32_t* offsets, void* h_ws, float* h_scale_ws,
                       int32_t* dev_status, cudaStream_t st, int nsm) {
  GemmPlan p;
  moe_status s = plan_gate_up(rows, H, w, a, a_scale, offsets, h_ws, h_scale_ws, dev_status, &p);
  return s != MOE_OK ? s : launch_plan(p, EPI_SWIGLU, st, nsm);
}

moe_status run_down(int32_t rows, int32_t H, const moe_ffn_weights* w, const void* h, const float* h_scale,
                    const int32_t* offsets, const float* row_w, void* out, int32_t* dev_status,
                    cudaStream_t st, int nsm) {
  GemmPlan p;
  moe_status s = plan_down(rows, H, w, h, h_scale, offsets, row_w, out, dev_status, &p);
  return s != MOE_OK ? s : launch_plan(p, EPI_WEIGHTED, st, nsm);
}


}  // namespace

extern "C" {

moe_status moe_gate_up_swiglu(int32_t rows, int32_t H, const moe_ffn_weights* w, const void* a,
                              const float* a_scale, const int32_t* offsets, void* h_ws, float* h_scale_ws,
                              int32_t* dev_status, void* stream) {
  moe_status s = check_ffn(rows, H, w, a, a_scale, true, false);
  if (s != MOE_OK) return s;
  if (!h_ws || (!offsets && w->groups != 1)) return MOE_ERR_INVALID_ARG;
  if (w->dtype == MOE_E4M3 && !h_scale_ws) return MOE_ERR_INVALID_ARG;
  if (any_misaligned(offsets, h_ws, h_scale_ws)) return MOE_ERR_ALIGNMENT;
  int nsm = 0;
  if ((s = sm_count(&nsm)) != MOE_OK) return s;
  return run_gate_up(rows, H, w, a, a_scale, offsets, h_ws, h_scale_ws, dev_status, as_stream(stream), nsm);
}

moe_status moe_gate_up_swiglu_gather(int32_t rows, int32_t H, const moe_ffn_weights* w, const void* x, int32_t T,
                                     const int32_t* src_token, const int32_t* offsets, void* h_ws,
                                     int32_t* dev_status, void* stream) {
  moe_status s = check_ffn(rows, H, w, x, nullptr, true, false);
  if (s != MOE_OK) return s;
  if (w->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (T < 1 || !src_token || !offsets || !h_ws) return MOE_ERR_INVALID_ARG;
  if (any_misaligned(src_token, offsets, h_ws)) return MOE_ERR_ALIGNMENT;
  int nsm = 0;
  if ((s = sm_count(&nsm)) != MOE_OK) return s;
  const int I = w->I;
  CUtensorMap tmA;
  TokenMaps tmB;
  s = w->tiled ? make_tmap(&tmA, w->w13, false, 64, static_cast<uint64_t>(w->groups) * 2 * I * (H / 64), 256)
               : make_tmap(&tmA, w->w13, false, H, static_cast<uint64_t>(w->groups) * 2 * I, 128);
  if (s != MOE_OK) return s;
  s = make_token_tmaps(&tmB, x, false, H, T);      // not read: token rows are gathered
  if (s != MOE_OK) return s;
  GemmArgs g1{};
  g1.rows = rows;
  g1.K = H;
  g1.groups = w->groups;
  g1.offsets = offsets;
  g1.a_rows_per_group = 2 * I;
  g1.a_tiled = w->tiled;
  g1.n_mblk = I / 128;
  g1.mblk_stride = 128;
  g1.sub1_off = I;
  g1.feat_stride = 128;
  g1.out = h_ws;
  g1.out_ld = I;
  g1.status = dev_status;
  g1.gather_src = x;
  g1.gather_rows = src_token;
  g1.gather_src_rows = T;
  g1.wait_ns = wait_limit();
  return check_launch(launch_grouped_gemm(false, EPI_SWIGLU, tmA, tmB, g1, nsm, as_stream(stream)));
}

moe_status moe_down_proj(int32_t rows, int32_t H, const moe_ffn_weights* w, const void* h, const float* h_scale,
                         const int32_t* offsets, const float* row_w, void* out, int32_t* dev_status,
                         void* stream) {
  moe_status s = check_ffn(rows, H, w, h, h_scale, false, true);
  if (s != MOE_OK) return s;
  if (!out || (!offsets && w->groups != 1)) return MOE_ERR_INVALID_ARG;
  if (any_misaligned(offsets, row_w, out)) return MOE_ERR_ALIGNMENT;
  int nsm = 0;
  if ((s = sm_count(&nsm)) != MOE_OK) return s;
  return run_down(rows, H, w, h, h_scale, offsets, row_w, out, dev_status, as_stream(stream), nsm);
}

moe_status moe_grouped_swiglu(int32_t rows, int32_t H, const moe_ffn_weights* w, const void* a,
                              const float* a_scale, const int32_t* offsets, const float* row_w,
                              void* h_ws, float* h_scale_ws, void* out, int32_t* dev_status, void* stream) {
  moe_status s = check_ffn(rows, H, w, a, a_scale, true, true);
  if (s != MOE_OK) return s;
  if (!h_ws || !out || (!offsets && w->groups != 1)) return MOE_ERR_INVALID_ARG;
  if (w->dtype == MOE_E4M3 && !h_scale_ws) return MOE_ERR_INVALID_ARG;
  if (any_misaligned(offsets, row_w, h_ws, h_scale_ws, out)) return MOE_ERR_ALIGNMENT;
  int nsm = 0;
  if ((s = sm_count(&nsm)) != MOE_OK) return s;
  cudaStream_t st = as_stream(stream);
  s = run_gate_up(rows, H, w, a, a_scale, offsets, h_ws, h_scale_ws, dev_status, st, nsm);
  if (s != MOE_OK) return s;
  return run_down(rows, H, w, h_ws, h_scale_ws, offsets, row_w, out, dev_status, st, nsm);
}

moe_status moe_gate_up_swiglu_with_shared(int32_t rows, int32_t H, const moe_ffn_weights* w, const void* a,
                                          const float* a_scale, const int32_t* offsets, void* h_ws,
                                          float* h_scale_ws, int32_t sh_rows, const moe_ffn_weights* sw,
                                          const void* sh_a, const float* sh_a_scale, void* sh_h_ws,
                                          float* sh_h_scale_ws, int32_t* dev_status, void* stream) {
  moe_status s = check_ffn(rows, H, w, a, a_scale, true, false);
  if (s != MOE_OK) return s;
  if ((s = check_ffn(sh_rows, H, sw, sh_a, sh_a_scale, true, false)) != MOE_OK) return s;
  if (!offsets || !h_ws || !sh_h_ws || sw->groups != 1 || sw->dtype != w->dtype) return MOE_ERR_INVALID_ARG;
  if (w->dtype == MOE_E4M3 && (!h_scale_ws || !sh_h_scale_ws)) return MOE_ERR_INVALID_ARG;
  if (any_misaligned(offsets, h_ws, h_scale_ws, sh_h_ws, sh_h_scale_ws)) return MOE_ERR_ALIGNMENT;
  int nsm = 0;
  if ((s = sm_count(&nsm)) != MOE_OK) return s;
  cudaStream_t st = as_stream(stream);
  GemmPlan p, q;
  if ((s = plan_gate_up(rows, H, w, a, a_scale, offsets, h_ws, h_scale_ws, dev_status, &p)) != MOE_OK) return s;
  if ((s = plan_gate_up(sh_rows, H, sw, sh_a, sh_a_scale, nullptr, sh_h_ws, sh_h_scale_ws, dev_status, &q)) !=
      MOE_OK)
    return s;
  return launch_plan(p, EPI_SWIGLU, st, nsm, &q);
}

moe_status moe_down_proj_with_shared(int32_t rows, int32_t H, const moe_ffn_weights* w, const void* h,
                                     const float* h_scale, const int32_t* offsets, const float* row_w, void* out,
                                     int32_t sh_rows, const moe_ffn_weights* sw, const void* sh_h,
                                     const float* sh_h_scale, void* sh_out, int32_t* dev_status, void* stream) {
  moe_status s = check_ffn(rows, H, w, h, h_scale, false, true);
  if (s != MOE_OK) return s;
  if ((s = check_ffn(sh_rows, H, sw, sh_h, sh_h_scale, false, true)) != MOE_OK) return s;
  if (!offsets || !out || !sh_out || sw->groups != 1 || sw->dtype != w->dtype) return MOE_ERR_INVALID_ARG;
  if (any_misaligned(offsets, row_w, out, sh_out)) return MOE_ERR_ALIGNMENT;
  int nsm = 0;
  if ((s = sm_count(&nsm)) != MOE_OK) return s;
  cudaStream_t st = as_stream(stream);
  GemmPlan p, q;
  if ((s = plan_down(rows, H, w, h, h_scale, offsets, row_w, out, dev_status, &p)) != MOE_OK) return s;
  if ((s = plan_down(sh_rows, H, sw, sh_h, sh_h_scale, nullptr, nullptr, sh_out, dev_status, &q)) != MOE_OK)
    return s;
  return launch_plan(p, EPI_WEIGHTED, st, nsm, &q);
}

moe_status moe_tile_ffn_weights(int32_t H, const moe_ffn_weights* src, void* w13_t, void* w2_t, void* stream) {
  if (!src || H < 1 || src->groups < 1 || src->I < 1 || src->tiled != 0) return MOE_ERR_INVALID_ARG;
  if (src->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (H % 256 != 0 || src->I % 128 != 0) return MOE_ERR_UNSUPPORTED;
  if (static_cast<long long>(src->groups) * 2 * src->I * (H / 64) > 0x7fffffffLL) return MOE_ERR_UNSUPPORTED;
  if ((w13_t && !src->w13) || (w2_t && !src->w2)) return MOE_ERR_INVALID_ARG;
  if (any_misaligned(src->w13, src->w2, w13_t, w2_t)) return MOE_ERR_ALIGNMENT;
  // the copies are gathers: an output overlapping any input would be read after being written
  const size_t b13 = static_cast<size_t>(src->groups) * 2 * src->I * H * 2, b2 = static_cast<size_t>(src->groups) * H * src->I * 2;
  auto overlap = [](const void* p, size_t np, const void* q, size_t nq) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(p), b = reinterpret_cast<uintptr_t>(q);
    return p && q && a < b + nq && b < a + np;
  };
  if (overlap(w13_t, b13, src->w13, b13) || overlap(w13_t, b13, src->w2, b2) || overlap(w2_t, b2, src->w13, b13) ||
      overlap(w2_t, b2, src->w2, b2) || overlap(w13_t, b13, w2_t, b2))
    return MOE_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  if (w13_t) {   // 256-row tiles: 128 gate rows, then the same features' 128 up rows
    moe_status s = check_launch(launch_tile_weights(src->w13, w13_t, src->groups, 2 * src->I, H, src->I, st));
    if (s != MOE_OK) return s;
  }
  if (w2_t) return check_launch(launch_tile_weights(src->w2, w2_t, src->groups, H, src->I, 0, st));
  return MOE_OK;
}

moe_status moe_swiglu_ffn_sync_size(int32_t rows, int32_t groups, int32_t sh_rows, size_t* bytes) {
  if (!bytes || rows < 1 || groups < 1 || sh_rows < 1) return MOE_ERR_INVALID_ARG;
  *bytes = sizeof(int32_t) * (ffn_routed_blocks(rows, groups) + ffn_blocks(sh_rows) + 1);
  return MOE_OK;
}

moe_status moe_swiglu_ffn_with_shared(int32_t rows, int32_t H, const moe_ffn_weights* w, const void* a,
                                      const int32_t* offsets, const float* row_w, void* h_ws, void* out,
                                      int32_t sh_rows, const moe_ffn_weights* sw, const void* sh_a, void* sh_h_ws,
                                      void* sh_out, void* sync_ws, size_t sync_ws_bytes, int32_t* dev_status,
                                      void* stream) {
  moe_status s = check_ffn(rows, H, w, a, nullptr, true, true);
  if (s != MOE_OK) return s;
  if ((s = check_ffn(sh_rows, H, sw, sh_a, nullptr, true, true)) != MOE_OK) return s;
  if (!offsets || !h_ws || !out || !sh_h_ws || !sh_out || !sync_ws || sw->groups != 1) return MOE_ERR_INVALID_ARG;
  if (w->dtype != MOE_BF16 || sw->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  const size_t nctr = ffn_routed_blocks(rows, w->groups) + ffn_blocks(sh_rows);
  const size_t need = sizeof(int32_t) * (nctr + 1);   // token-block counters, then the tile counter
  if (sync_ws_bytes < need) return MOE_ERR_INVALID_ARG;
  if (any_misaligned(offsets, row_w, h_ws, out, sh_h_ws, sh_out, sync_ws)) return MOE_ERR_ALIGNMENT;
  int nsm = 0;
  if ((s = sm_count(&nsm)) != MOE_OK) return s;
  cudaStream_t st = as_stream(stream);
  GemmPlan gu, sgu, dn, sdn;
  if ((s = plan_gate_up(sh_rows, H, sw, sh_a, nullptr, nullptr, sh_h_ws, nullptr, dev_status, &sgu)) != MOE_OK)
    return s;
  if ((s = plan_gate_up(rows, H, w, a, nullptr, offsets, h_ws, nullptr, dev_status, &gu)) != MOE_OK) return s;
  if ((s = plan_down(sh_rows, H, sw, sh_h_ws, nullptr, nullptr, nullptr, sh_out, dev_status, &sdn)) != MOE_OK)
    return s;
  if ((s = plan_down(rows, H, w, h_ws, nullptr, offsets, row_w, out, dev_status, &dn)) != MOE_OK) return s;
  FfnArgs f{};
  const GemmPlan* plans[4] = {&sgu, &gu, &sdn, &dn};
  for (int i = 0; i < 4; ++i) {
    f.tmA[i] = plans[i]->tmA;
    f.tmB[i] = plans[i]->tmB;
    f.g[i] = plans[i]->g;
  }
  f.ready = static_cast<int32_t*>(sync_ws);
  f.tile_counter = f.ready + nctr;
  f.shared_base = ffn_routed_blocks(rows, w->groups);
  cudaError_t e = cudaMemsetAsync(sync_ws, 0, need, st);
  if (e != cudaSuccess) return cuda_fail(e);
  return check_launch(launch_ffn_bf16(f, nsm, st));
}

moe_status moe_down_proj_combine(int32_t rows, int32_t T, int32_t H, const moe_ffn_weights* w, const void* h,
                                 const int32_t* offsets, const float* row_w, const int32_t* src_token,
                                 const moe_ffn_weights* sw, const void* sh_h, float* acc_ws, void* y,
                                 int32_t* dev_status, void* stream) {
  moe_status s = check_ffn(rows, H, w, h, nullptr, false, true);
  if (s != MOE_OK) return s;
  if (w->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (T < 1 || !offsets || !row_w || !src_token || !acc_ws || !y) return MOE_ERR_INVALID_ARG;
  if (sw) {
    if ((s = check_ffn(T, H, sw, sh_h, nullptr, false, true)) != MOE_OK) return s;
    if (sw->groups != 1 || sw->dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
  }
  if (any_misaligned(offsets, row_w, src_token, acc_ws, y)) return MOE_ERR_ALIGNMENT;
  int nsm = 0;
  if ((s = sm_count(&nsm)) != MOE_OK) return s;
  cudaStream_t st = as_stream(stream);
  cudaError_t e = cudaMemsetAsync(acc_ws, 0, static_cast<size_t>(T) * H * sizeof(float), st);
  if (e != cudaSuccess) return cuda_fail(e);
  GemmPlan p, q;
  if ((s = plan_down(rows, H, w, h, nullptr, offsets, row_w, acc_ws, dev_status, &p)) != MOE_OK) return s;
  p.g.scatter_tok = src_token;
  p.g.scatter_T = T;
  if (sw) {
    if ((s = plan_down(T, H, sw, sh_h, nullptr, nullptr, nullptr, acc_ws, dev_status, &q)) != MOE_OK) return s;
    q.g.scatter_tok = nullptr;
    q.g.scatter_T = T;
  }
  if ((s = launch_plan(p, EPI_SCATTER, st, nsm, sw ? &q : nullptr)) != MOE_OK) return s;
  return check_launch(launch_cast_rows(T, H, acc_ws, y, st));
}

moe_status moe_combine(int32_t T, int32_t k, int32_t H, const void* expert_out, const int32_t* slot_to_row,
                       const float* topk_w, const void* shared_out, void* y, void* stream) {
  if (T < 1 || k < 1 || H < 1 || !expert_out || !slot_to_row || !y) return MOE_ERR_INVALID_ARG;
  if (k > 16 || H % 8 != 0) return MOE_ERR_UNSUPPORTED;
  if (any_misaligned(expert_out, slot_to_row, topk_w, shared_out, y)) return MOE_ERR_ALIGNMENT;
  return check_launch(launch_combine(T, k, H, expert_out, slot_to_row, topk_w, shared_out, y, as_stream(stream)));
}

moe_status moe_bias_update(int32_t E, int32_t T, int32_t k, const int32_t* expert_counts, float* bias,
                           float gamma, float* load_cv, void* stream) {
  if (E < 1 || T < 1 || k < 1 || !expert_counts || !bias) return MOE_ERR_INVALID_ARG;
  if (E > 1024) return MOE_ERR_UNSUPPORTED;
  if (any_misaligned(expert_counts, bias, load_cv)) return MOE_ERR_ALIGNMENT;
  return check_launch(launch_bias_update(E, T, k, expert_counts, bias, gamma, load_cv, as_stream(stream)));
}

moe_status moe_aux_loss_workspace_size(int32_t T, int32_t E, int32_t seq_len, size_t* bytes) {
  if (!bytes || T < 1 || E < 1 || seq_len < 1 || T % seq_len != 0) return MOE_ERR_INVALID_ARG;
  *bytes = aux_loss_workspace_bytes(T, E, seq_len);
  return MOE_OK;
}

moe_status moe_aux_loss(int32_t T, int32_t E, int32_t k, int32_t seq_len, int32_t scoring, const float* logits,
                        const int32_t* topk_ids, float alpha, float* aux_out, void* workspace,
                        size_t workspace_bytes, int32_t* dev_status, void* stream) {
  if (T < 1 || E < 1 || k < 1 || k > E || seq_len < 1 || T % seq_len != 0) return MOE_ERR_INVALID_ARG;
  if (scoring != MOE_SOFTMAX && scoring != MOE_SIGMOID) return MOE_ERR_INVALID_ARG;
  if (!logits || !topk_ids || !aux_out || !workspace) return MOE_ERR_INVALID_ARG;
  if (workspace_bytes < aux_loss_workspace_bytes(T, E, seq_len)) return MOE_ERR_INVALID_ARG;
  if (E > 256) return MOE_ERR_UNSUPPORTED;
  if (reinterpret_cast<uintptr_t>(workspace) % 8 != 0 || reinterpret_cast<uintptr_t>(logits) % 4 != 0 ||
      reinterpret_cast<uintptr_t>(topk_ids) % 4 != 0 || reinterpret_cast<uintptr_t>(aux_out) % 4 != 0)
    return MOE_ERR_ALIGNMENT;
  return check_launch(launch_aux_loss(T, E, k, seq_len, scoring, logits, topk_ids, alpha, aux_out, workspace,
                                      dev_status, as_stream(stream)));
}

moe_status moe_quantize_blocks(int32_t batch, int32_t N, int32_t K, const void* w, void* q, float* scale,
                               void* stream) {
  if (batch < 1 || N < 1 || K < 1 || !w || !q || !scale) return MOE_ERR_INVALID_ARG;
  if (N % 128 != 0 || K % 128 != 0 || batch > 65535 || N / 128 > 65535) return MOE_ERR_UNSUPPORTED;
  if (any_misaligned(w, q, scale)) return MOE_ERR_ALIGNMENT;
  return check_launch(launch_quant_blocks(batch, N, K, w, q, scale, as_stream(stream)));
}

moe_status moe_quantize_rows(int32_t M, int32_t K, const void* a, void* q, float* scale, void* stream) {
  if (M < 1 || K < 1 || !a || !q || !scale) return MOE_ERR_INVALID_ARG;
  if (K % 128 != 0) return MOE_ERR_UNSUPPORTED;
  if (any_misaligned(a, q, scale)) return MOE_ERR_ALIGNMENT;
  return check_launch(launch_quant_rows(M, K, a, q, scale, as_stream(stream)));
}

moe_status moe_read_device_status(const int32_t* dev_status, int32_t* out, void* stream) {
  if (!dev_status || !out) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  int32_t v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, dev_status, sizeof(v), cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) return cuda_fail(e);
  e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e);
  *out = v;
  if (v == 0) return MOE_OK;
  if (v == MOE_DEVSTAT_TIMEOUT) return MOE_ERR_DEVICE_TIMEOUT;
  return MOE_ERR_DEVICE_CHECK;
}

}  // extern "C"
