// Token permutation into per-expert contiguous segments.
//
// "MoE 混合专家模型推理参数与前向传播详解" §3.2: every token is copied once per
// chosen expert and the copies are laid out expert by expert; the worked
// example there orders each expert's segment by ascending token index and
// gives expert_first_token_offset as the segment boundaries. That is a stable
// counting sort of the T*k (token, slot) pairs keyed by expert, done here in
// four launches:
//   1. perm_hist  : per block of kTokBlock tokens, an expert histogram;
//   2. perm_scan  : expert offsets (exclusive scan of the totals) and, per
//                   block, the first row of each expert's part of the segment;
//   3. perm_rank  : per block, one warp walks the slots in token order and
//                   gives each its row (warp match on equal experts ranks the
//                   32 slots of a step at once);
//   4. perm_copy  : one warp per token reads the token's row once and writes
//                   it to its k rows with 16-byte vector loads and stores
//                   (fp8 rows also carry their 1x128 scales).
#include "kernels.cuh"

namespace moe {

constexpr int kTokBlock = 64;        // tokens per rank block

__global__ void perm_hist_kernel(const int32_t* __restrict__ ids, int T, int k, int E,
                                 int32_t* __restrict__ blockhist, int32_t* status) {
  extern __shared__ int hist_dyn[];
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist_dyn[e] = 0;
  __syncthreads();
  const int s0 = blockIdx.x * kTokBlock * k;
  const int s1 = min(T, (blockIdx.x + 1) * kTokBlock) * k;
  for (int s = s0 + threadIdx.x; s < s1; s += blockDim.x) {
    const int e = ids[s];
    if (e >= 0 && e < E) atomicAdd(&hist_dyn[e], 1);
    else flag_status(status, MOE_DEVSTAT_BAD_EXPERT_ID);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    blockhist[static_cast<size_t>(blockIdx.x) * E + e] = hist_dyn[e];
}

// One CTA of 1024 threads. Thread (e, part) owns expert e for blocks
// [part*nb/parts, (part+1)*nb/parts).
__global__ void __launch_bounds__(1024)
perm_scan_kernel(int32_t* __restrict__ blockhist, int nb, int E, int total,
                 int32_t* __restrict__ offsets) {
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
  if (active) {
    int s = 0;
    for (int b = b0; b < b1; ++b) s += blockhist[static_cast<size_t>(b) * E + e];
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
    for (int b = b0; b < b1; ++b) {
      const size_t i = static_cast<size_t>(b) * E + e;
      const int c = blockhist[i];
      blockhist[i] = run;
      run += c;
    }
  }
}

// One warp per block of kTokBlock tokens.
__global__ void __launch_bounds__(32)
perm_rank_kernel(const int32_t* __restrict__ ids, const float* __restrict__ topk_w, int T, int k,
                 int E, const int32_t* __restrict__ blockbase, int32_t* __restrict__ slot_to_row,
                 int32_t* __restrict__ src_token, float* __restrict__ row_w) {
  extern __shared__ int cnt[];
  const int lane = threadIdx.x;
  for (int e = lane; e < E; e += 32) cnt[e] = blockbase[static_cast<size_t>(blockIdx.x) * E + e];
  __syncwarp();
  const int s0 = blockIdx.x * kTokBlock * k;
  const int s1 = min(T, (blockIdx.x + 1) * kTokBlock) * k;
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int base = s0; base < s1; base += 32) {
    const int s = base + lane;
    int e = -1;
    if (s < s1) {
      e = ids[s];
      if (e < 0 || e >= E) e = -2 - lane;   // unique key: never grouped, never counted
    } else {
      e = -2 - lane;
    }
    const unsigned grp = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(grp & lt_mask);
    const bool valid = e >= 0;
    const int base_row = valid ? cnt[e] : 0;
    __syncwarp();
    if (valid && lane == 31 - __clz(grp)) cnt[e] = base_row + __popc(grp);
    __syncwarp();
    if (valid) {
      const int r = base_row + rank;
      slot_to_row[s] = r;
      src_token[r] = s / k;
      if (row_w) row_w[r] = topk_w[s];
    } else if (s < s1) {
      slot_to_row[s] = -1;                   // id out of range (flagged by perm_hist)
    }
  }
}

// One warp per token: x[t] -> x_perm[slot_to_row[t*k + j]] for j < k.
constexpr int kPermKMax = 16;

__global__ void __launch_bounds__(256)
perm_copy_kernel(const uint4* __restrict__ x, int T, int k, int vec_per_row,
                 const int32_t* __restrict__ slot_to_row, uint4* __restrict__ x_perm,
                 const float* __restrict__ x_scale, float* __restrict__ x_perm_scale, int nscale) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;                                  // warp-uniform
  const int nrows = T * k;
  int my_row = lane < k ? slot_to_row[static_cast<size_t>(t) * k + lane] : -1;
  if (my_row >= nrows) my_row = -1;                   // never write outside x_perm
  int rows[kPermKMax];
#pragma unroll
  for (int j = 0; j < kPermKMax; ++j) rows[j] = __shfl_sync(0xffffffffu, my_row, j);
  const uint4* src = x + static_cast<size_t>(t) * vec_per_row;
  for (int base = 0; base < vec_per_row; base += 128) {   // same trip count on every lane
    uint4 val[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int v = base + u * 32 + lane;
      if (v < vec_per_row) val[u] = __ldg(src + v);
    }
#pragma unroll
    for (int j = 0; j < kPermKMax; ++j) {
      if (j < k && rows[j] >= 0) {
        uint4* dst = x_perm + static_cast<size_t>(rows[j]) * vec_per_row;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int v = base + u * 32 + lane;
          if (v < vec_per_row) dst[v] = val[u];
        }
      }
    }
  }
  if (x_scale) {
    for (int i = lane; i < nscale; i += 32) {
      const float sc = x_scale[static_cast<size_t>(t) * nscale + i];
#pragma unroll
      for (int j = 0; j < kPermKMax; ++j)
        if (j < k && rows[j] >= 0) x_perm_scale[static_cast<size_t>(rows[j]) * nscale + i] = sc;
    }
  }
}

size_t permute_workspace_bytes(int T, int E) {
  const int nb = (T + kTokBlock - 1) / kTokBlock;
  return static_cast<size_t>(nb) * E * sizeof(int32_t);
}

cudaError_t launch_permute(int T, int k, int E, int row_bytes, const int32_t* ids, const float* topk_w,
                           const void* x, const float* x_scale, int nscale, void* x_perm,
                           float* x_perm_scale, int32_t* offsets, int32_t* src_token,
                           int32_t* slot_to_row, float* row_w, int32_t* blockhist, int32_t* status,
                           cudaStream_t stream) {
  const int nb = (T + kTokBlock - 1) / kTokBlock;
  perm_hist_kernel<<<nb, 256, E * sizeof(int), stream>>>(ids, T, k, E, blockhist, status);
  const int parts = 1024 / E;
  const size_t scan_smem = (static_cast<size_t>(parts) * E + E + 32) * sizeof(int);
  perm_scan_kernel<<<1, 1024, scan_smem, stream>>>(blockhist, nb, E, T * k, offsets);
  perm_rank_kernel<<<nb, 32, E * sizeof(int), stream>>>(ids, topk_w, T, k, E, blockhist, slot_to_row,
                                                       src_token, row_w);
  if (x_perm) {
    const int warps = 8;
    perm_copy_kernel<<<(T + warps - 1) / warps, warps * 32, 0, stream>>>(
        reinterpret_cast<const uint4*>(x), T, k, row_bytes / 16, slot_to_row,
        reinterpret_cast<uint4*>(x_perm), x_scale, x_perm_scale, nscale);
  }
  return cudaGetLastError();
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
  return moe_permute(T, k, E, H, topk_ids, topk_w, x, x_dtype, x_scale, x_perm, x_perm_scale, expert_offsets,
                     src_token, slot_to_row, row_w, ws, kStaticWsBytes, dev_status, stream);
}
