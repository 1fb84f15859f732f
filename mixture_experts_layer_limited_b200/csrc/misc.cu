// Combine, aux-loss-free bias update and E4M3 quantisers.
#include "kernels.cuh"

namespace moe {

__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float (&f)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 p = __bfloat1622float2(h[i]);
    f[2 * i] = p.x;
    f[2 * i + 1] = p.y;
  }
}

__device__ __forceinline__ uint4 f32_to_bf16x8(const float (&f)[8]) {
  uint4 v;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
  return v;
}

// Unpermute + weighted combine ("MoE 混合专家模型推理参数与前向传播详解" §3.4):
// y[t] = shared[t] + sum_j w[t][j] * expert_out[slot_to_row[t*k+j]], fp32 sum in
// slot order, one bf16 rounding. One warp per token, two 16-byte vectors per
// lane and step so 2k row loads are in flight. KMAX >= k bounds the rows
// held in registers.
template <int KMAX>
__global__ void __launch_bounds__(256)
combine_kernel(int T, int k, int vec_per_row, const uint4* __restrict__ eo,
               const int32_t* __restrict__ slot_to_row, const float* __restrict__ topk_w,
               const uint4* __restrict__ shared, uint4* __restrict__ y) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;                       // warp-uniform
  const int nrows = T * k;
  int my_row = lane < k ? slot_to_row[static_cast<size_t>(t) * k + lane] : -1;
  if (my_row >= nrows) my_row = -1;
  const float my_w = (lane < k && topk_w) ? topk_w[static_cast<size_t>(t) * k + lane] : 1.0f;
  int rows[KMAX];
  float ws[KMAX];
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    rows[j] = __shfl_sync(0xffffffffu, my_row, j);
    ws[j] = __shfl_sync(0xffffffffu, my_w, j);
  }
  const uint4* sh = shared ? shared + static_cast<size_t>(t) * vec_per_row : nullptr;
  uint4* yt = y + static_cast<size_t>(t) * vec_per_row;
  for (int base = 0; base < vec_per_row; base += 64) {
    const int v0 = base + lane, v1 = base + 32 + lane;
    const bool ok0 = v0 < vec_per_row, ok1 = v1 < vec_per_row;
    uint4 r0[KMAX], r1[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      if (j < k && rows[j] >= 0) {
        const uint4* src = eo + static_cast<size_t>(rows[j]) * vec_per_row;
        if (ok0) r0[j] = __ldcs(src + v0);
        if (ok1) r1[j] = __ldcs(src + v1);
      }
    }
    float a0[8], a1[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) { a0[i] = 0.0f; a1[i] = 0.0f; }
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      if (j < k && rows[j] >= 0) {
        float f0[8], f1[8];
        bf16x8_to_f32(r0[j], f0);
        bf16x8_to_f32(r1[j], f1);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          a0[i] += ws[j] * f0[i];
          a1[i] += ws[j] * f1[i];
        }
      }
    }
    if (sh) {
      float f0[8], f1[8];
      if (ok0) bf16x8_to_f32(__ldg(sh + v0), f0);
      if (ok1) bf16x8_to_f32(__ldg(sh + v1), f1);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (ok0) a0[i] += f0[i];
        if (ok1) a1[i] += f1[i];
      }
    }
    if (ok0) yt[v0] = f32_to_bf16x8(a0);
    if (ok1) yt[v1] = f32_to_bf16x8(a1);
  }
}

// Aux-loss-free bias step (xxqk.cn digest §2.2): overloaded experts' bias
// down by gamma, underloaded up, compared with the mean load exactly.
// Optional load CV = sample std / mean (gsyq.cn teardown §4).
__global__ void __launch_bounds__(1024)
bias_update_kernel(int E, int T, int k, const int32_t* __restrict__ counts, float* __restrict__ bias,
                   float gamma, float* __restrict__ load_cv) {
  __shared__ double red[32];
  __shared__ double mean_s;
  const int e = threadIdx.x;
  const long long c = e < E ? static_cast<long long>(counts[e]) : 0;
  if (e < E) {
    const long long d = c * E - static_cast<long long>(T) * k;
    const float s = d > 0 ? 1.0f : (d < 0 ? -1.0f : 0.0f);
    bias[e] = bias[e] - gamma * s;
  }
  if (!load_cv) return;                     // block-uniform
  const int lane = e & 31, warp = e >> 5;
  double v = static_cast<double>(c);
  for (int d = 16; d > 0; d >>= 1) v += __shfl_xor_sync(0xffffffffu, v, d);
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (e == 0) {
    double s = 0.0;
    for (int w = 0; w < 32; ++w) s += red[w];
    mean_s = s / E;
  }
  __syncthreads();
  const double dm = e < E ? static_cast<double>(c) - mean_s : 0.0;
  v = dm * dm;
  for (int d = 16; d > 0; d >>= 1) v += __shfl_xor_sync(0xffffffffu, v, d);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (e == 0) {
    double s = 0.0;
    for (int w = 0; w < 32; ++w) s += red[w];
    const double sd = E > 1 ? sqrt(s / (E - 1)) : 0.0;
    *load_cv = static_cast<float>(mean_s > 0.0 ? sd / mean_s : 0.0);
  }
}

// ------------------------------------------------------------------------
// Sequence-level auxiliary balance loss ("MoE 混合专家模型推理参数与前向传播详解"
// §6.2): per sequence E * sum_e f_e * P_e, f_e = the expert's share of the
// sequence's seq_len * k assignments, P_e = mean normalised score.
// Pass 1, one CTA per chunk of <= kAuxChunk tokens inside one sequence: warp w
// takes tokens w, w + 8, ...; lane l keeps the fp64 score sums of experts
// l, l + 32, ...; the eight warps' sums are added in warp order and the chunk's
// sums and assignment counts go to the workspace.
// Pass 2, one CTA: per expert, chunks in order, sum_b count_be * P_be; then a
// fixed tree over experts. Deterministic for given inputs.
// ------------------------------------------------------------------------
__global__ void __launch_bounds__(kAuxWarps * 32)
aux_chunk_kernel(int T, int E, int k, int seq_len, int scoring, const float* __restrict__ logits,
                 const int32_t* __restrict__ ids, double* __restrict__ psum, int32_t* __restrict__ cnt,
                 int32_t* status) {
  __shared__ double part[kAuxWarps][256];
  __shared__ int hist[256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cps = (seq_len + kAuxChunk - 1) / kAuxChunk;          // chunks per sequence
  const int seq = blockIdx.x / cps, c = blockIdx.x % cps;
  const int t0 = seq * seq_len + c * kAuxChunk;
  const int t1 = min(t0 + kAuxChunk, (seq + 1) * seq_len);
  for (int e = threadIdx.x; e < 256; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  double acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.0;
  for (int t = t0 + warp; t < t1; t += kAuxWarps) {
    const float* L = logits + static_cast<size_t>(t) * E;
    double z[8];
    double m = -INFINITY;
    if (scoring == MOE_SOFTMAX) {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (lane + 32 * i < E) m = fmax(m, static_cast<double>(L[lane + 32 * i]));
#pragma unroll
      for (int d = 16; d > 0; d >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, d));
    }
    double sum = 0.0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane + 32 * i;
      z[i] = 0.0;
      if (e < E) {
        const double l = static_cast<double>(L[e]);
        z[i] = scoring == MOE_SOFTMAX ? exp(l - m) : 1.0 / (1.0 + exp(-l));
      }
      sum += z[i];
    }
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, d);
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] += z[i] / sum;
    if (lane < k) {
      const int e = ids[static_cast<size_t>(t) * k + lane];
      if (e >= 0 && e < E) atomicAdd(&hist[e], 1);
      else flag_status(status, MOE_DEVSTAT_BAD_EXPERT_ID);
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) part[warp][lane + 32 * i] = acc[i];
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    double v = 0.0;
    for (int w = 0; w < kAuxWarps; ++w) v += part[w][e];
    psum[static_cast<size_t>(blockIdx.x) * E + e] = v;
    cnt[static_cast<size_t>(blockIdx.x) * E + e] = hist[e];
  }
}

__global__ void __launch_bounds__(256)
aux_reduce_kernel(int E, int k, int seq_len, int n_seq, int cps, float alpha, const double* __restrict__ psum,
                  const int32_t* __restrict__ cnt, float* __restrict__ out) {
  __shared__ double red[256];
  const int e = threadIdx.x;
  double v = 0.0;
  if (e < E) {
    for (int b = 0; b < n_seq; ++b) {
      double p = 0.0;
      long long n = 0;
      for (int c = 0; c < cps; ++c) {
        const size_t i = (static_cast<size_t>(b) * cps + c) * E + e;
        p += psum[i];
        n += cnt[i];
      }
      v += static_cast<double>(n) * p;
    }
  }
  red[e] = v;
  __syncthreads();
  for (int s = 128; s > 0; s >>= 1) {
    if (e < s) red[e] += red[e + s];
    __syncthreads();
  }
  if (e == 0) {
    const double S = static_cast<double>(seq_len);
    *out = static_cast<float>(static_cast<double>(alpha) * E * red[0] / (static_cast<double>(n_seq) * S * S * k));
  }
}

// E4M3 weight quantisation per 128x128 block. grid (K/128, N/128, batch),
// 256 threads: thread i covers row i/2, columns (i%2)*64 .. +64.
__global__ void __launch_bounds__(256)
quant_blocks_kernel(const __nv_bfloat16* __restrict__ w, int N, int K, uint8_t* __restrict__ q,
                    float* __restrict__ scale) {
  __shared__ float red[8];
  const int i = threadIdx.x;
  const size_t b = blockIdx.z;
  const int r = blockIdx.y * 128 + (i >> 1);
  const int c0 = blockIdx.x * 128 + (i & 1) * 64;
  const size_t off = b * static_cast<size_t>(N) * K + static_cast<size_t>(r) * K + c0;
  const uint4* src = reinterpret_cast<const uint4*>(w + off);
  float f[64];
  float amax = 0.0f;
#pragma unroll
  for (int v = 0; v < 8; ++v) {
    float t[8];
    bf16x8_to_f32(src[v], t);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      f[v * 8 + j] = t[j];
      amax = fmaxf(amax, fabsf(t[j]));
    }
  }
  for (int d = 16; d > 0; d >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, d));
  if ((i & 31) == 0) red[i >> 5] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int j = 1; j < 8; ++j) amax = fmaxf(amax, red[j]);
  const float sc = amax == 0.0f ? 1.0f : amax / 448.0f;
  uint32_t packed[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    packed[j] = static_cast<uint32_t>(to_e4m3(f[4 * j] / sc)) |
                (static_cast<uint32_t>(to_e4m3(f[4 * j + 1] / sc)) << 8) |
                (static_cast<uint32_t>(to_e4m3(f[4 * j + 2] / sc)) << 16) |
                (static_cast<uint32_t>(to_e4m3(f[4 * j + 3] / sc)) << 24);
  }
  uint4* dst = reinterpret_cast<uint4*>(q + off);
#pragma unroll
  for (int j = 0; j < 4; ++j) dst[j] = make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
  if (i == 0) scale[(b * (N / 128) + blockIdx.y) * (K / 128) + blockIdx.x] = sc;
}

// E4M3 activation quantisation per 1x128 tile: one warp per tile, 4 values a lane.
__global__ void __launch_bounds__(256)
quant_rows_kernel(const __nv_bfloat16* __restrict__ a, int M, int K, uint8_t* __restrict__ q,
                  float* __restrict__ scale) {
  const int lane = threadIdx.x & 31;
  const long long tile = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int nkb = K / 128;
  if (tile >= static_cast<long long>(M) * nkb) return;   // warp-uniform
  const long long m = tile / nkb;
  const int kb = static_cast<int>(tile - m * nkb);
  const size_t off = static_cast<size_t>(m) * K + kb * 128 + lane * 4;
  const uint2 raw = *reinterpret_cast<const uint2*>(a + off);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
  const float2 p0 = __bfloat1622float2(h[0]), p1 = __bfloat1622float2(h[1]);
  float amax = fmaxf(fmaxf(fabsf(p0.x), fabsf(p0.y)), fmaxf(fabsf(p1.x), fabsf(p1.y)));
  for (int d = 16; d > 0; d >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, d));
  const float sc = amax == 0.0f ? 1.0f : amax / 448.0f;
  const uint32_t packed = static_cast<uint32_t>(to_e4m3(p0.x / sc)) |
                          (static_cast<uint32_t>(to_e4m3(p0.y / sc)) << 8) |
                          (static_cast<uint32_t>(to_e4m3(p1.x / sc)) << 16) |
                          (static_cast<uint32_t>(to_e4m3(p1.y / sc)) << 24);
  *reinterpret_cast<uint32_t*>(q + off) = packed;
  if (lane == 0) scale[m * nkb + kb] = sc;
}

// ------------------------------------------------------------------------
cudaError_t launch_combine(int T, int k, int H, const void* eo, const int32_t* slot_to_row,
                           const float* topk_w, const void* shared, void* y, cudaStream_t stream) {
  const int warps = 8;
  const dim3 grid((T + warps - 1) / warps), block(warps * 32);
  const uint4* e = reinterpret_cast<const uint4*>(eo);
  const uint4* sh = reinterpret_cast<const uint4*>(shared);
  uint4* out = reinterpret_cast<uint4*>(y);
  if (k <= 4) combine_kernel<4><<<grid, block, 0, stream>>>(T, k, H / 8, e, slot_to_row, topk_w, sh, out);
  else if (k <= 8) combine_kernel<8><<<grid, block, 0, stream>>>(T, k, H / 8, e, slot_to_row, topk_w, sh, out);
  else combine_kernel<16><<<grid, block, 0, stream>>>(T, k, H / 8, e, slot_to_row, topk_w, sh, out);
  return cudaGetLastError();
}

// y[t] = bf16(acc[t]) for the fp32 accumulator of the combine fused into the
// down GEMM; 8 elements (32 B in, 16 B out) per thread, streamed.
__global__ void __launch_bounds__(256)
cast_rows_kernel(const float4* __restrict__ acc, uint4* __restrict__ y, size_t n8) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const float4 a = __ldcs(acc + 2 * i), b = __ldcs(acc + 2 * i + 1);
    __nv_bfloat162 p0 = __floats2bfloat162_rn(a.x, a.y), p1 = __floats2bfloat162_rn(a.z, a.w);
    __nv_bfloat162 p2 = __floats2bfloat162_rn(b.x, b.y), p3 = __floats2bfloat162_rn(b.z, b.w);
    uint4 o;
    o.x = *reinterpret_cast<uint32_t*>(&p0);
    o.y = *reinterpret_cast<uint32_t*>(&p1);
    o.z = *reinterpret_cast<uint32_t*>(&p2);
    o.w = *reinterpret_cast<uint32_t*>(&p3);
    y[i] = o;
  }
}

cudaError_t launch_cast_rows(int T, int H, const float* acc, void* y, cudaStream_t stream) {
  const size_t n8 = static_cast<size_t>(T) * H / 8;
  const size_t blocks = (n8 + 255) / 256;
  cast_rows_kernel<<<static_cast<unsigned>(blocks < 148 * 8 ? blocks : 148 * 8), 256, 0, stream>>>(
      reinterpret_cast<const float4*>(acc), reinterpret_cast<uint4*>(y), n8);
  return cudaGetLastError();
}

cudaError_t launch_bias_update(int E, int T, int k, const int32_t* counts, float* bias, float gamma,
                               float* load_cv, cudaStream_t stream) {
  bias_update_kernel<<<1, 1024, 0, stream>>>(E, T, k, counts, bias, gamma, load_cv);
  return cudaGetLastError();
}

cudaError_t launch_aux_loss(int T, int E, int k, int seq_len, int scoring, const float* logits,
                            const int32_t* ids, float alpha, float* out, void* ws, int32_t* status,
                            cudaStream_t stream) {
  const int n_seq = T / seq_len;
  const int cps = (seq_len + kAuxChunk - 1) / kAuxChunk;
  const long long chunks = static_cast<long long>(n_seq) * cps;
  double* psum = reinterpret_cast<double*>(ws);
  int32_t* cnt = reinterpret_cast<int32_t*>(psum + chunks * E);
  aux_chunk_kernel<<<static_cast<unsigned>(chunks), kAuxWarps * 32, 0, stream>>>(
      T, E, k, seq_len, scoring, logits, ids, psum, cnt, status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  aux_reduce_kernel<<<1, 256, 0, stream>>>(E, k, seq_len, n_seq, cps, alpha, psum, cnt, out);
  return cudaGetLastError();
}

cudaError_t launch_quant_blocks(int batch, int N, int K, const void* w, void* q, float* scale,
                                cudaStream_t stream) {
  dim3 grid(K / 128, N / 128, batch);
  quant_blocks_kernel<<<grid, 256, 0, stream>>>(reinterpret_cast<const __nv_bfloat16*>(w), N, K,
                                                reinterpret_cast<uint8_t*>(q), scale);
  return cudaGetLastError();
}

cudaError_t launch_quant_rows(int M, int K, const void* a, void* q, float* scale, cudaStream_t stream) {
  const long long tiles = static_cast<long long>(M) * (K / 128);
  const int warps = 8;
  const long long blocks = (tiles + warps - 1) / warps;
  quant_rows_kernel<<<static_cast<unsigned>(blocks), warps * 32, 0, stream>>>(
      reinterpret_cast<const __nv_bfloat16*>(a), M, K, reinterpret_cast<uint8_t*>(q), scale);
  return cudaGetLastError();
}

// ------------------------------------------------------------------------
// Weight tiling (moe_tile_ffn_weights): one thread per 16-byte chunk of the
// output, each tile 256 rows x 64 columns (32 KB) of one group's weights.
// ------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
tile_weights_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, size_t chunks, int M, int K, int split) {
  const int nkb = K / 64;
  const int nblk = split ? M / 256 : 0;   // 256-row tiles per group when they interleave two halves
  for (size_t d = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; d < chunks;
       d += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t tile = d / (256 * 8);
    const int within = static_cast<int>(d - tile * (256 * 8));
    const int r = within >> 3, c16 = within & 7;
    const size_t kb = tile % nkb, blk = tile / nkb;      // blk = g * (M / 256) + row block
    size_t row;
    if (split) {   // rows [0, 128): block rows of the first half; [128, 256): the same of the second
      const size_t g = blk / nblk, f = blk % nblk;
      row = g * M + f * 128 + (r >= 128 ? split : 0) + (r & 127);
    } else {
      row = blk * 256 + r;
    }
    dst[d] = src[row * static_cast<size_t>(K / 8) + kb * 8 + c16];
  }
}

// dst tile t = (g * (M / 256) + b) * (K / 64) + kb holds, at rows t * 256 of a
// [*, 64] matrix, the 64 columns kb of 256 source rows of group g: rows b * 256
// + [0, 256) (split = 0), or rows b * 128 + [0, 128) followed by split + b * 128
// + [0, 128) (gate/up weights, split = I).
cudaError_t launch_tile_weights(const void* src, void* dst, int G, int M, int K, int split, cudaStream_t stream) {
  const size_t chunks = static_cast<size_t>(G) * M * (K / 8);
  const size_t blocks = (chunks + 255) / 256;
  const int grid = static_cast<int>(blocks < 65535 * 16 ? blocks : 65535 * 16);
  tile_weights_kernel<<<grid, 256, 0, stream>>>(static_cast<const uint4*>(src), static_cast<uint4*>(dst), chunks, M, K,
                                                split);
  return cudaGetLastError();
}

}  // namespace moe
