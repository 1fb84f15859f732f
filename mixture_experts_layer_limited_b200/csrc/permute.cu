// Token permutation into per-expert contiguous segments.
//
// "MoE 混合专家模型推理参数与前向传播详解" §3.2: every token is copied once per
// chosen expert and the copies are laid out expert by expert; the worked
// example there orders each expert's segment by ascending token index and
// gives expert_first_token_offset as the segment boundaries. That is a stable
// counting sort of the T*k (token, slot) pairs keyed by expert, done here in
// three launches:
//   1. perm_hist  : per block of kTokBlock tokens, an expert histogram and
//                   each slot's rank among the block's slots of its expert
//                   (kept in slot_to_row until step 3 replaces it);
//   2. perm_scan  : expert offsets (exclusive scan of the totals) and, per
//                   block, the first row of each expert's part of the segment;
//   3. perm_place : one warp per token adds the two for each of its slots,
//                   writes the metadata, reads the token's row once and
//                   writes it to its k rows.

#include "kernels.cuh"

namespace moe {

constexpr int kTokBlock = 64;        // tokens per rank block

// 256 threads; the block's slots (token-major, then slot) are taken 256 at a
// time in order. A slot's rank = its expert's count over the earlier passes
// + the counts of the earlier warps of this pass + the earlier lanes of its
// own warp with the same expert (match_any), so equal experts keep slot
// order: the stable sort's order inside the block.
constexpr int kHistThreads = 256;

__global__ void __launch_bounds__(kHistThreads)
perm_hist_kernel(const int32_t* __restrict__ ids, int T, int k, int E, int32_t* __restrict__ blockhist,
                 int32_t* __restrict__ local_rank, int32_t* status) {
  griddep_launch_dependents();                         // the scan may be scheduled now
  constexpr int kWarps = kHistThreads / 32;
  extern __shared__ int hist_dyn[];
  int* cnt = hist_dyn;                                  // [E]: the earlier passes' slots per expert
  int* wcnt = hist_dyn + E;                             // [kWarps][E]: this pass's slots per warp and expert
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int e = threadIdx.x; e < E; e += kHistThreads) cnt[e] = 0;
  const int s0 = blockIdx.x * kTokBlock * k;
  const int s1 = min(T, (blockIdx.x + 1) * kTokBlock) * k;
  for (int base = s0; base < s1; base += kHistThreads) {   // same trip count in the whole CTA
    for (int i = threadIdx.x; i < kWarps * E; i += kHistThreads) wcnt[i] = 0;
    __syncthreads();
    const int s = base + threadIdx.x;
    int e = -1;
    if (s < s1) {
      e = ids[s];
      if (e < 0 || e >= E) {
        flag_status(status, MOE_DEVSTAT_BAD_EXPERT_ID);
        e = -1;
      }
    }
    const uint32_t peers = __match_any_sync(0xffffffffu, e);
    const int intra = __popc(peers & ((1u << lane) - 1u));
    if (e >= 0 && intra == 0) wcnt[warp * E + e] = __popc(peers);
    __syncthreads();
    if (e >= 0) {
      int rank = cnt[e] + intra;
      for (int w = 0; w < warp; ++w) rank += wcnt[w * E + e];
      local_rank[s] = rank;
    } else if (s < s1) {
      local_rank[s] = -1;
    }
    __syncthreads();                                    // cnt read before it advances
    for (int x = threadIdx.x; x < E; x += kHistThreads) {
      int add = 0;
      for (int w = 0; w < kWarps; ++w) add += wcnt[w * E + x];
      cnt[x] += add;
    }
    __syncthreads();                                    // wcnt read before the next pass clears it
  }
  for (int e = threadIdx.x; e < E; e += kHistThreads)
    blockhist[static_cast<size_t>(blockIdx.x) * E + e] = cnt[e];
}

// One CTA of 1024 threads. Thread (e, part) owns expert e for blocks
// [part*nb/parts, (part+1)*nb/parts).
__global__ void __launch_bounds__(1024)
perm_scan_kernel(int32_t* __restrict__ blockhist, int nb, int E, int total,
                 int32_t* __restrict__ offsets) {
  griddep_wait();                                      // the histograms are complete
  griddep_launch_dependents();                         // the copy kernel's CTAs may start their row loads
  extern __shared__ int sdyn[];
  const int parts = blockDim.x / E;                 // >= 1 (E <= 1024)
  int* part_sum = sdyn;                             // [parts][E]
  int* tot = sdyn + parts * E;                      // [E]
  int* warp_tot = tot + E;                          // [32]
  const int tid = threadIdx.x;
  const int e = tid % E, part = tid / E;
  const bool active = part < parts;
  const int per = (nb + parts - 1) / parts;
  const int b0 = min(nb, part * per), b1 = min(nb, b0 + per);
  constexpr int kChunk = 16;                        // independent loads in flight per thread
  if (active) {
    int s = 0;
    for (int c = b0; c < b1; c += kChunk) {
      int v[kChunk];
#pragma unroll
      for (int i = 0; i < kChunk; ++i) v[i] = c + i < b1 ? blockhist[static_cast<size_t>(c + i) * E + e] : 0;
#pragma unroll
      for (int i = 0; i < kChunk; ++i) s += v[i];
    }
    part_sum[part * E + e] = s;
  }
  __syncthreads();
  // totals and exclusive scan over experts (threads 0..E-1)
  int my_tot = 0;
  if (tid < E) {
    for (int p = 0; p < parts; ++p) my_tot += part_sum[p * E + tid];
  }
  int incl = my_tot;
  const int lane = tid & 31, warp = tid >> 5;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += v;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = warp_tot[lane];
    int wi = w;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, wi, d);
      if (lane >= d) wi += v;
    }
    warp_tot[lane] = wi - w;                        // exclusive
  }
  __syncthreads();
  if (tid < E) {
    const int excl = warp_tot[warp] + incl - my_tot;
    tot[tid] = excl;
    offsets[tid] = excl;
    if (tid == E - 1) offsets[E] = total;
  }
  __syncthreads();
  // rewrite blockhist in place as the first row of (block, expert)
  if (active) {
    int run = tot[e];
    for (int p = 0; p < part; ++p) run += part_sum[p * E + e];
    for (int c = b0; c < b1; c += kChunk) {
      int v[kChunk];
#pragma unroll
      for (int i = 0; i < kChunk; ++i) v[i] = c + i < b1 ? blockhist[static_cast<size_t>(c + i) * E + e] : 0;
#pragma unroll
      for (int i = 0; i < kChunk; ++i) {
        if (c + i < b1) blockhist[static_cast<size_t>(c + i) * E + e] = run;
        run += v[i];
      }
    }
  }
}

// One warp per token t: its rows, then the copies.
//   row of slot (t, j) = first row of (block of t, expert e) from perm_scan
//                        + the slot's rank inside the block from perm_hist
// (token order, then slot order: the stable counting sort). Lane j < k
// writes slot j's slot_to_row / src_token / row_w; the warp reads the token's
// row once and writes it to its k rows with 16-byte vector loads and stores
// (fp8 rows also carry their 1x128 scales). Slots with ids outside [0, E)
// get row -1 (flagged by perm_hist) and are not written.
constexpr int kPermKMax = 16;

// The rows of token t's k slots (lane j < k returns slot j's row, -1 for an
// invalid id) and their metadata; slot_to_row holds perm_hist's ranks on
// entry and the rows on return.
__device__ __forceinline__ int perm_rows_of_token(int t, int lane, const int32_t* __restrict__ ids,
                                                  const float* __restrict__ topk_w, int T, int k, int E,
                                                  const int32_t* __restrict__ blockbase,
                                                  int32_t* __restrict__ slot_to_row,
                                                  int32_t* __restrict__ src_token, float* __restrict__ row_w) {
  const int nrows = T * k;
  const int b = t / kTokBlock;
  const size_t s = static_cast<size_t>(t) * k + lane;
  int my_row = -1;
  if (lane < k) {
    const int e = ids[s];
    const int rank = slot_to_row[s];
    if (e >= 0 && e < E && rank >= 0) {
      my_row = blockbase[static_cast<size_t>(b) * E + e] + rank;
      if (my_row >= nrows) my_row = -1;                 // never write outside the rows
    }
    slot_to_row[s] = my_row;
    if (my_row >= 0) {
      src_token[my_row] = t;
      if (row_w) row_w[my_row] = topk_w[s];
    }
  }
  return my_row;
}

__global__ void __launch_bounds__(256, 3)
perm_place_kernel(const int32_t* __restrict__ ids, const float* __restrict__ topk_w, int T, int k, int E,
                  const int32_t* __restrict__ blockbase, int32_t* __restrict__ slot_to_row,
                  int32_t* __restrict__ src_token, float* __restrict__ row_w,
                  const uint4* __restrict__ x, int vec_per_row, uint4* __restrict__ x_perm,
                  const float* __restrict__ x_scale, float* __restrict__ x_perm_scale, int nscale) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;                                  // warp-uniform
  const uint4* src = x + static_cast<size_t>(t) * vec_per_row;
  uint4 val[8];
  if (x_perm) {                                        // the row's first chunk in flight during the metadata
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int v = u * 32 + lane;
      if (v < vec_per_row) val[u] = __ldg(src + v);
    }
  }
  griddep_wait();                                      // ranks and first rows complete
  const int my_row = perm_rows_of_token(t, lane, ids, topk_w, T, k, E, blockbase, slot_to_row, src_token, row_w);
  if (!x_perm) return;                                 // metadata only
  for (int base = 0; base < vec_per_row; base += 256) {   // same trip count on every lane
    if (base > 0) {
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int v = base + u * 32 + lane;
        if (v < vec_per_row) val[u] = __ldg(src + v);
      }
    }
#pragma unroll
    for (int j = 0; j < kPermKMax; ++j) {
      if (j >= k) break;                                  // warp-uniform
      const int row = __shfl_sync(0xffffffffu, my_row, j);   // the row of slot j (lane j holds it)
      if (row >= 0) {
        uint4* dst = x_perm + static_cast<size_t>(row) * vec_per_row;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int v = base + u * 32 + lane;
          if (v < vec_per_row) __stcs(dst + v, val[u]);        // streamed: x_perm is far larger than L2
        }
      }
    }
  }
  if (x_scale) {
    for (int j = 0; j < k; ++j) {
      const int row = __shfl_sync(0xffffffffu, my_row, j);
      if (row < 0) continue;                              // warp-uniform
      for (int i = lane; i < nscale; i += 32)
        x_perm_scale[static_cast<size_t>(row) * nscale + i] = x_scale[static_cast<size_t>(t) * nscale + i];
    }
  }
}

// bf16 rows quantised to E4M3 on their way to the k rows (x_perm E4M3):
// per 1x128 tile along H, scale = amax / 448 (1 for an all-zero tile) and
// code = RNE-saturated E4M3 of v / scale, both IEEE fp32 (the FP8 inference
// post's 1x128 dynamic activation tiles; the same bytes as
// moe_quantize_rows). Lane l holds 16 consecutive values of the row, 8 lanes
// one tile, so a warp step covers 4 tiles and every store is 16 bytes. x_q /
// x_q_scale (optional) receive the token's own codes and scales, unpermuted.
__global__ void __launch_bounds__(256, 3)
perm_place_quant_kernel(const int32_t* __restrict__ ids, const float* __restrict__ topk_w, int T, int k, int E,
                        const int32_t* __restrict__ blockbase, int32_t* __restrict__ slot_to_row,
                        int32_t* __restrict__ src_token, float* __restrict__ row_w,
                        const __nv_bfloat16* __restrict__ x, int H, uint8_t* __restrict__ x_perm,
                        float* __restrict__ x_perm_scale, uint8_t* __restrict__ x_q,
                        float* __restrict__ x_q_scale) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;                                  // warp-uniform
  griddep_wait();                                      // ranks and first rows complete
  const int my_row = perm_rows_of_token(t, lane, ids, topk_w, T, k, E, blockbase, slot_to_row, src_token, row_w);
  if (!x_perm && !x_q) return;                         // metadata only
  const int ntiles = H / 128;
  const __nv_bfloat16* src = x + static_cast<size_t>(t) * H;
  for (int tb = 0; tb < ntiles; tb += 4) {             // same trip count on every lane
    const int tile = tb + (lane >> 3);
    const bool valid = tile < ntiles;                  // uniform within each 8-lane group
    const int e0 = tile * 128 + (lane & 7) * 16;
    float v[16];
    if (valid) {
      const uint4 r0 = __ldg(reinterpret_cast<const uint4*>(src + e0));
      const uint4 r1 = __ldg(reinterpret_cast<const uint4*>(src + e0 + 8));
      const __nv_bfloat162* h0 = reinterpret_cast<const __nv_bfloat162*>(&r0);
      const __nv_bfloat162* h1 = reinterpret_cast<const __nv_bfloat162*>(&r1);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 a = __bfloat1622float2(h0[i]), b = __bfloat1622float2(h1[i]);
        v[2 * i] = a.x;
        v[2 * i + 1] = a.y;
        v[8 + 2 * i] = b.x;
        v[8 + 2 * i + 1] = b.y;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = 0.0f;
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
    for (int d = 4; d > 0; d >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, d));
    const float sc = amax == 0.0f ? 1.0f : amax / 448.0f;
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      w[i] = static_cast<uint32_t>(to_e4m3(v[4 * i] / sc)) | (static_cast<uint32_t>(to_e4m3(v[4 * i + 1] / sc)) << 8) |
             (static_cast<uint32_t>(to_e4m3(v[4 * i + 2] / sc)) << 16) |
             (static_cast<uint32_t>(to_e4m3(v[4 * i + 3] / sc)) << 24);
    const uint4 codes = make_uint4(w[0], w[1], w[2], w[3]);
    if (x_perm) {
#pragma unroll
      for (int j = 0; j < kPermKMax; ++j) {
        if (j >= k) break;                               // warp-uniform
        const int row = __shfl_sync(0xffffffffu, my_row, j);
        if (row >= 0 && valid) {
          *reinterpret_cast<uint4*>(x_perm + static_cast<size_t>(row) * H + e0) = codes;
          if ((lane & 7) == 0) x_perm_scale[static_cast<size_t>(row) * ntiles + tile] = sc;
        }
      }
    }
    if (x_q && valid) {
      *reinterpret_cast<uint4*>(x_q + static_cast<size_t>(t) * H + e0) = codes;
      if ((lane & 7) == 0) x_q_scale[static_cast<size_t>(t) * ntiles + tile] = sc;
    }
  }
}

// Launches kern as a programmatic dependent of the kernel before it in the
// stream (see griddep_wait).
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                             Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
  return e != cudaSuccess ? e : cudaGetLastError();
}

size_t permute_workspace_bytes(int T, int E) {   // blockhist[nb][E]
  const int nb = (T + kTokBlock - 1) / kTokBlock;
  return static_cast<size_t>(nb) * E * sizeof(int32_t);
}

cudaError_t launch_permute(int T, int k, int E, int H, bool x_e4m3, bool perm_e4m3, const int32_t* ids,
                           const float* topk_w, const void* x, const float* x_scale, void* x_perm,
                           float* x_perm_scale, void* x_q, float* x_q_scale, int32_t* offsets,
                           int32_t* src_token, int32_t* slot_to_row, float* row_w, int32_t* blockhist,
                           int32_t* status, cudaStream_t stream) {
  const int nb = (T + kTokBlock - 1) / kTokBlock;
  perm_hist_kernel<<<nb, kHistThreads, (kHistThreads / 32 + 1) * E * sizeof(int), stream>>>(
      ids, T, k, E, blockhist, slot_to_row, status);
  const int parts = 1024 / E;
  const size_t scan_smem = (static_cast<size_t>(parts) * E + E + 32) * sizeof(int);
  // the scan and the copy kernel are launched as programmatic dependents: each
  // may be scheduled before the kernel ahead of it ends, and waits for it
  // (griddep_wait) before reading its output; the copy kernel's row loads,
  // which need none, start during the scan
  cudaError_t e = launch_dependent(perm_scan_kernel, dim3(1), dim3(1024), scan_smem, stream, blockhist, nb, E,
                                   T * k, offsets);
  if (e != cudaSuccess) return e;
  const int warps = 8;
  const dim3 grid((T + warps - 1) / warps), block(warps * 32);
  if (!x_e4m3 && perm_e4m3)
    return launch_dependent(perm_place_quant_kernel, grid, block, 0, stream, ids, topk_w, T, k, E,
                            static_cast<const int32_t*>(blockhist), slot_to_row, src_token, row_w,
                            static_cast<const __nv_bfloat16*>(x), H, static_cast<uint8_t*>(x_perm), x_perm_scale,
                            static_cast<uint8_t*>(x_q), x_q_scale);
  const int row_bytes = x_e4m3 ? H : 2 * H;
  return launch_dependent(perm_place_kernel, grid, block, 0, stream, ids, topk_w, T, k, E,
                          static_cast<const int32_t*>(blockhist), slot_to_row, src_token, row_w,
                          reinterpret_cast<const uint4*>(x), row_bytes / 16, reinterpret_cast<uint4*>(x_perm),
                          x_e4m3 ? x_scale : static_cast<const float*>(nullptr), x_perm_scale, H / 128);
}

}  // namespace moe

// ------------------------------------------------------------------------
// moe_permute_static_ws: the permutation with its scratch in this library's
// own device memory, for callers that cannot allocate (see include/moe.h).
// ------------------------------------------------------------------------
#include <mutex>

namespace {

constexpr size_t kStaticWsBytes = size_t(1) << 20;      // 1 MiB
constexpr int kMaxDevices = 64;

// The scratch itself: one copy per device that loads the library. In host
// code this name is only a stand-in for the symbol; its device address comes
// from cudaGetSymbolAddress below.
__device__ __align__(256) int32_t g_permute_static_ws[kStaticWsBytes / sizeof(int32_t)];

std::mutex g_static_ws_mu;
void* g_static_ws_ptr[kMaxDevices] = {};

}  // namespace

extern "C" moe_status moe_permute_static_ws(int32_t T, int32_t k, int32_t E, int32_t H,
                                            const int32_t* topk_ids, const float* topk_w,
                                            const void* x, moe_dtype x_dtype, const float* x_scale,
                                            void* x_perm, float* x_perm_scale, int32_t* expert_offsets,
                                            int32_t* src_token, int32_t* slot_to_row, float* row_w,
                                            int32_t* dev_status, void* stream) {
  if (T < 1 || k < 1 || E < 1) return MOE_ERR_INVALID_ARG;
  if (moe::permute_workspace_bytes(T, E) > kStaticWsBytes) return MOE_ERR_UNSUPPORTED;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  void* ws = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_static_ws_mu);
    if (!g_static_ws_ptr[dev]) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_permute_static_ws) != cudaSuccess || p == nullptr) return MOE_ERR_CUDA;
      g_static_ws_ptr[dev] = p;
    }
    ws = g_static_ws_ptr[dev];
  }
  return moe_permute(T, k, E, H, topk_ids, topk_w, x, x_dtype, x_scale, x_perm, x_dtype, x_perm_scale, nullptr,
                     nullptr, expert_offsets, src_token, slot_to_row, row_w, ws, kStaticWsBytes, dev_status,
                     stream);
}
