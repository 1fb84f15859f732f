// Argument blocks and launchers shared by the kernels and the C-ABI layer.
#pragma once

#include "common.cuh"

namespace moe {

struct GemmArgs {
  int32_t rows = 0;                // activation rows (B operand)
  int32_t K = 0;                   // reduction length
  int32_t groups = 1;              // number of segments
  const int32_t* offsets = nullptr;  // [groups + 1] or nullptr (one segment)
  int32_t a_rows_per_group = 0;    // weight rows per group (2I or H)
  int32_t n_mblk = 0;              // weight blocks per group
  int32_t mblk_stride = 0;         // weight-row stride between blocks (128 / 256)
  int32_t sub1_off = 0;            // weight-row offset of sub-tile 1 (I / 128)
  int32_t feat_stride = 0;         // output-feature stride between blocks (128 / 256)
  int32_t feat_sub1 = 0;           // output-feature offset of sub-tile 1 (0 / 128)
  int32_t bn_max = 256;            // max tokens per tile (multiple of 32, <= 256)
  int32_t a_one_box = 0;           // a tile's 256 weight rows are contiguous: one TMA box
  int32_t a_tiled = 0;             // weights in moe_tile_ffn_weights' layout: a tile's 256 rows of K block kb at
                                   // row ((g * n_mblk + mb) * nk + kb) * 256 of a [*, 64] matrix
  void* out = nullptr;             // [rows, out_ld] bf16, or e4m3 codes (GEMM1 FP8)
  int32_t out_ld = 0;
  const float* row_w = nullptr;    // [rows] or nullptr
  const float* a_scale = nullptr;  // E4M3: [groups, a_rows_per_group/128, K/128]
  const float* b_scale = nullptr;  // E4M3: [rows, K/128]
  float* out_scale = nullptr;      // E4M3 GEMM1: [rows, out_ld/128]
  int32_t* status = nullptr;
  // Gathered token rows (gate/up GEMM of the routed experts): B row p is
  // row gather_rows[p] of gather_src [*, K] instead of row p of the B map.
  const void* gather_src = nullptr;
  const int32_t* gather_rows = nullptr;
  int32_t gather_src_rows = 0;     // rows of gather_src (indices outside [0, this) are flagged, not read)
  int32_t epi_warps = 4;           // bf16 kernel: epilogue warps (4 or 12)
  // EPI_SCATTER: token of each row ([rows], NULL: the row is the token) and the
  // number of tokens (rows of the fp32 accumulator `out`)
  const int32_t* scatter_tok = nullptr;
  int32_t scatter_T = 0;
  uint64_t wait_ns = kDefaultWaitLimitNs;  // limit of each bounded mbarrier wait
};

struct RouteArgs {
  int32_t T, H, E, k, G, g;
  int32_t scoring, norm;
  float scale;
  const float* bias;        // [E] or nullptr
  float* logits;            // [T, E] (out for the GEMM kernel when non-null, in for the other)
  int32_t* ids;             // [T, k]
  float* w;                 // [T, k]
  int32_t* counts;          // [E], zeroed beforehand
  int32_t* status;
  uint64_t wait_ns;         // limit of each bounded mbarrier wait
};

// EPI_SCATTER: GEMM2 with the combine fused in: the weighted fp32 rows are
// added atomically into a [tokens, H] fp32 accumulator at their token.
enum { EPI_SWIGLU = 0, EPI_WEIGHTED = 1, EPI_SCATTER = 2 };

// Token-row tensor maps: bf16 boxes of 256, 128, 64, 32 and 16 rows (a tile's
// rows are fetched with the fewest boxes); e4m3 uses box[0] of 32 rows.
constexpr int kTokBoxes = 5;
struct TokenMaps {
  CUtensorMap box[kTokBoxes];
};

// A second single-group problem for the same launch (bf16).
struct SecondProblem {
  CUtensorMap tmA;
  TokenMaps tmB;
  GemmArgs a;
};
cudaError_t launch_grouped_gemm(bool e4m3, int epi, const CUtensorMap& tmA, const TokenMaps& tmB,
                                const GemmArgs& a, int grid, cudaStream_t stream,
                                const SecondProblem* two = nullptr);

// Both bf16 GEMMs of the SwiGLU experts, routed and shared, in one persistent
// launch: g[0] shared gate/up, g[1] routed gate/up, g[2] shared down, g[3]
// routed down (g[1] and g[3] share offsets; all four bn_max = 256). ready:
// one int32 counter per token block, zeroed before the launch: routed token
// blocks from 0, the shared problem's from shared_base; tile_counter: the
// next tile to hand out, zeroed before the launch.
struct FfnArgs {
  CUtensorMap tmA[4];
  TokenMaps tmB[4];
  GemmArgs g[4];
  int32_t* ready;
  int32_t* tile_counter;
  int32_t shared_base;
};
static_assert(sizeof(FfnArgs) <= 4096, "FfnArgs must fit the kernel parameter space");
constexpr int kFfnEpiWarps = 12;
constexpr int kGuQ = 1;       // epilogue warps per TMEM lane quarter on the gate/up tiles
cudaError_t launch_ffn_bf16(const FfnArgs& f, int grid, cudaStream_t stream);
// w [G, M, K] bf16 row-major -> tiles of R rows x 64 K, tile (g*(M/R) + rb, kb)
// at rows ((g*(M/R) + rb)*(K/64) + kb)*R of a [*, 64] matrix
cudaError_t launch_tile_weights(const void* src, void* dst, int G, int M, int K, int split, cudaStream_t stream);
// route: also route the tokens in the same launch where the shape allows
// (route8_experts_per_thread(r) > 0); counts must be zeroed beforehand. The
// split of the hidden size over a cluster's CTAs depends on T and num_sms only,
// so the logits of a given T are the same with and without routing.
cudaError_t launch_gate_gemm(const CUtensorMap& tmX, const CUtensorMap& tmG, const RouteArgs& r, bool route,
                             int num_sms, cudaStream_t stream);
int route8_experts_per_thread(const RouteArgs& r);
cudaError_t launch_route_tokens(const RouteArgs& r, int num_sms, cudaStream_t stream);
size_t permute_workspace_bytes(int T, int E);
// x_e4m3: x holds E4M3 codes (+ x_scale); perm_e4m3: x_perm receives codes
// (+ x_perm_scale), quantised here when x is bf16 (x_q / x_q_scale, optional,
// then also receive the token's own codes).
cudaError_t launch_permute(int T, int k, int E, int H, bool x_e4m3, bool perm_e4m3, const int32_t* ids,
                           const float* topk_w, const void* x, const float* x_scale, void* x_perm,
                           float* x_perm_scale, void* x_q, float* x_q_scale, int32_t* offsets,
                           int32_t* src_token, int32_t* slot_to_row, float* row_w, int32_t* blockhist,
                           int32_t* status, cudaStream_t stream);
cudaError_t launch_combine(int T, int k, int H, const void* eo, const int32_t* slot_to_row,
                           const float* topk_w, const void* shared, void* y, cudaStream_t stream);
constexpr int kAuxChunk = 128;   // tokens per aux-loss partial
constexpr int kAuxWarps = 8;
inline size_t aux_loss_workspace_bytes(int T, int E, int seq_len) {
  const size_t chunks = static_cast<size_t>(T / seq_len) * ((seq_len + kAuxChunk - 1) / kAuxChunk);
  return chunks * E * (sizeof(double) + sizeof(int32_t));
}
cudaError_t launch_aux_loss(int T, int E, int k, int seq_len, int scoring, const float* logits,
                            const int32_t* ids, float alpha, float* out, void* ws, int32_t* status,
                            cudaStream_t stream);
cudaError_t launch_cast_rows(int T, int H, const float* acc, void* y, cudaStream_t stream);
cudaError_t launch_bias_update(int E, int T, int k, const int32_t* counts, float* bias, float gamma,
                               float* load_cv, cudaStream_t stream);
cudaError_t launch_quant_blocks(int batch, int N, int K, const void* w, void* q, float* scale,
                                cudaStream_t stream);
cudaError_t launch_quant_rows(int M, int K, const void* a, void* q, float* scale, cudaStream_t stream);

}  // namespace moe
