// Router: gate projection, scoring, group-limited top-k, routing weights.
//
// Pages: "MoE 混合专家模型推理参数与前向传播详解" §2.1 (router_logits =
// hidden_states @ gate.weight^T) and §3.1 (softmax scoring, greedy top-k, no
// renormalisation for V2-Lite); the gsyq.cn DeepSeek-V3 teardown §3-§4 (sigmoid
// scoring plus a balancing bias, n_group = 8 groups scored by the sum of their
// top-2, topk_group = 4 kept, top-8 within, renormalise, x routed_scaling_factor);
// the xxqk.cn digest §2.2 (bias only steers selection; device-limited routing).
//
// Kernel 1 (route_gemm_kernel): one CTA per 128 tokens. The gate GEMM runs on
// tcgen05 (M = 128 tokens, N = E experts, K = H) with TMA-fed operands and an
// fp32 accumulator of 128 x E in TMEM. Each of the 128 epilogue threads owns
// one TMEM lane = one token and routes it alone: the E logits are pulled out of
// TMEM 32 at a time, scored into a per-thread shared-memory column (reusing the
// operand ring), and the group scores / top-k are kept in registers. No
// cross-thread communication is needed except the per-CTA expert histogram.
// Kernel 2 (route_logits_kernel): same routing from fp32 logits in memory.
#include "kernels.cuh"

namespace moe {

constexpr int kRouteKMax = 16;
constexpr int kRouteRows = 128;     // tokens per CTA = scratch column count
constexpr int kRouteMaxGroups = 32;



// Score -> fp32 as the library states it: sigmoid in double, rounded once.
__device__ __forceinline__ float sigmoid_rn(float v) {
  return static_cast<float>(1.0 / (1.0 + exp(-static_cast<double>(v))));
}

// Routes the token whose scratch column is `col` (expert e at col[e * 128];
// holds fp32 sigmoid for sigmoid scoring, the raw logit for softmax).
__device__ void route_token(const float* col, float* gcol, const float* bias_s, float lmax,
                            double sumexp, const RouteArgs& c, int32_t* ids_out, float* w_out,
                            int* hist) {
  const bool sig = c.scoring == MOE_SIGMOID;
  const bool raw_logit = !sig && c.G == 1 && bias_s == nullptr;
  auto sel = [&](int e) -> float {
    const float v = col[e * kRouteRows];
    if (sig) return bias_s ? v + bias_s[e] : v;
    if (raw_logit) return v;
    const float p = static_cast<float>(exp(static_cast<double>(v) - static_cast<double>(lmax)) / sumexp);
    return bias_s ? p + bias_s[e] : p;
  };
  const int gsz = c.E / c.G;
  uint32_t kept = 0xffffffffu;
  if (c.G > 1) {
    for (int gi = 0; gi < c.G; ++gi) {
      float m1 = -INFINITY, m2 = -INFINITY;
      for (int e = gi * gsz; e < (gi + 1) * gsz; ++e) {
        const float v = sel(e);
        if (v > m1) { m2 = m1; m1 = v; } else if (v > m2) { m2 = v; }
      }
      gcol[gi * kRouteRows] = gsz >= 2 ? m1 + m2 : m1;
    }
    kept = 0;
    for (int r = 0; r < c.g; ++r) {
      float best = -INFINITY;
      int bi = -1;
      for (int gi = 0; gi < c.G; ++gi) {
        if ((kept >> gi) & 1u) continue;
        const float v = gcol[gi * kRouteRows];
        if (bi < 0 || v > best) { best = v; bi = gi; }
      }
      kept |= 1u << bi;
    }
  }
  float tv[kRouteKMax];
  int ti[kRouteKMax];
#pragma unroll
  for (int s = 0; s < kRouteKMax; ++s) { tv[s] = -INFINITY; ti[s] = 0; }
  for (int gi = 0; gi < c.G; ++gi) {
    if (!((kept >> gi) & 1u)) continue;
    for (int e = gi * gsz; e < (gi + 1) * gsz; ++e) {
      const float v = sel(e);
      // insert keeping (value desc, index asc); equal values never displace
#pragma unroll
      for (int s = kRouteKMax - 1; s >= 0; --s) {
        if (s < c.k && v > tv[s]) {
          if (s > 0 && v > tv[s > 0 ? s - 1 : 0]) {
            tv[s] = tv[s > 0 ? s - 1 : 0];
            ti[s] = ti[s > 0 ? s - 1 : 0];
          } else {
            tv[s] = v;
            ti[s] = e;
          }
        }
      }
    }
  }
  float w[kRouteKMax];
  float sum = 0.0f;
#pragma unroll
  for (int s = 0; s < kRouteKMax; ++s) {
    if (s < c.k) {
      const float v = col[ti[s] * kRouteRows];
      w[s] = sig ? v : static_cast<float>(exp(static_cast<double>(v) - static_cast<double>(lmax)) / sumexp);
      sum += w[s];
    }
  }
#pragma unroll
  for (int s = 0; s < kRouteKMax; ++s) {
    if (s < c.k) {
      float ws = c.norm ? w[s] / sum : w[s];
      ids_out[s] = ti[s];
      w_out[s] = ws * c.scale;
      atomicAdd(&hist[ti[s]], 1);
    }
  }
}

// Per-token scoring pass over an E-wide logit row delivered 32 at a time.
struct ScorePass {
  float lmax = -INFINITY;
  __device__ __forceinline__ void chunk(float* col, const float (&v)[32], int e0, int E, bool sig) {
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      if (e0 + j < E) {
        col[(e0 + j) * kRouteRows] = sig ? sigmoid_rn(v[j]) : v[j];
        lmax = fmaxf(lmax, v[j]);
      }
    }
  }
};

__device__ __forceinline__ double softmax_denominator(const float* col, int E, float lmax) {
  double s = 0.0;
  for (int e = 0; e < E; ++e) s += exp(static_cast<double>(col[e * kRouteRows]) - static_cast<double>(lmax));
  return s;
}

size_t route_scratch_bytes(int E) {
  return static_cast<size_t>(kRouteRows) * (E + kRouteMaxGroups) * sizeof(float);
}

// ------------------------------------------------------------------------
// Kernel 1: fused tcgen05 gate GEMM + routing.
// ------------------------------------------------------------------------
constexpr int kRouteStages = 4;

__global__ void __launch_bounds__(192, 1)
route_gemm_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmG,
                  const RouteArgs r, uint32_t tmem_cols) {
  constexpr int KB = 64;
  extern __shared__ __align__(1024) uint8_t dsmem[];
  __shared__ uint64_t full_bar[kRouteStages], empty_bar[kRouteStages];
  __shared__ uint64_t tmem_full, drain_bar, epi_bar;
  __shared__ uint32_t tmem_base_s;
  __shared__ int issued_parity[kRouteStages];
  __shared__ volatile int abort_flag;
  __shared__ int hist[256];
  __shared__ float bias_s[256];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
  const uint32_t a_bytes = 128u * 128u;
  const uint32_t b_bytes = static_cast<uint32_t>(r.E) * 128u;
  const uint32_t stage_bytes = a_bytes + b_bytes;
  const int m0 = blockIdx.x * kRouteRows;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kRouteStages; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 1);
      issued_parity[i] = -1;
    }
    mbar_init(&tmem_full, 1);
    mbar_init(&drain_bar, 1);
    mbar_init(&epi_bar, 128);
    abort_flag = 0;
    fence_barrier_init();
  }
  for (int e = threadIdx.x; e < r.E; e += blockDim.x) {
    hist[e] = 0;
    bias_s[e] = r.bias ? r.bias[e] : 0.0f;
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmG);
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_s, tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_s;
  const int nk = r.H / KB;

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol_x = policy_evict_first();
      const uint64_t pol_g = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      for (int kb = 0; kb < nk; ++kb) {
        if (!mbar_wait(&empty_bar[stage], phase ^ 1u, &abort_flag, r.status)) break;
        mbar_arrive_expect_tx(&full_bar[stage], stage_bytes);
        uint8_t* st = smem + stage * stage_bytes;
        tma_load_2d(st, &tmX, &full_bar[stage], kb * KB, m0, pol_x);
        tma_load_2d(st + a_bytes, &tmG, &full_bar[stage], kb * KB, 0, pol_g);
        issued_parity[stage] = static_cast<int>(phase);
        if (++stage == kRouteStages) { stage = 0; phase ^= 1u; }
      }
      if (abort_flag) {
        for (int i = 0; i < kRouteStages; ++i)
          if (issued_parity[i] >= 0) mbar_wait_drain(&full_bar[i], static_cast<uint32_t>(issued_parity[i]));
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = make_idesc(1u, 128u, static_cast<uint32_t>(r.E));
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int kb = 0; kb < nk; ++kb) {
        if (!mbar_wait(&full_bar[stage], phase, &abort_flag, r.status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a0 = smem_u32(smem + stage * stage_bytes);
        const uint32_t b0 = a0 + a_bytes;
#pragma unroll
        for (int kk = 0; kk < KB / 16; ++kk)
          umma_bf16(tmem_base, sw128_desc(a0 + kk * 32), sw128_desc(b0 + kk * 32), idesc, (kb | kk) != 0);
        umma_commit(&empty_bar[stage]);
        if (++stage == kRouteStages) { stage = 0; phase ^= 1u; }
      }
      if (ok) umma_commit(&tmem_full);
      umma_commit(&drain_bar);
      mbar_wait_drain(&drain_bar, 0);
    }
  } else {
    const int q = warp & 3;
    const int row = 32 * q + lane;           // TMEM lane == token row in tile
    const int tok = m0 + row;
    bool ok = mbar_wait(&tmem_full, 0, &abort_flag, r.status);
    if (ok) {
      tc_fence_after();
      float* scratch = reinterpret_cast<float*>(smem);   // operand ring is idle now
      float* col = scratch + row;
      float* gcol = scratch + static_cast<size_t>(kRouteRows) * r.E + row;
      const bool sig = r.scoring == MOE_SIGMOID;
      ScorePass sp;
      const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(32 * q) << 16);
      for (int c = 0; c * 32 < r.E; ++c) {
        float v[32];
        tmem_ld32(lane_addr + c * 32, v);
        tmem_ld_wait();
        if (tok < r.T) {
          if (r.logits) {
            float4* dst = reinterpret_cast<float4*>(r.logits + static_cast<size_t>(tok) * r.E + c * 32);
#pragma unroll
            for (int j = 0; j < 8; ++j)
              if (c * 32 + 4 * j < r.E) dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
          }
          sp.chunk(col, v, c * 32, r.E, sig);
        }
      }
      tc_fence_before();
      if (tok < r.T) {
        const double den = sig ? 1.0 : softmax_denominator(col, r.E, sp.lmax);
        route_token(col, gcol, r.bias ? bias_s : nullptr, sp.lmax, den, r,
                    r.ids + static_cast<size_t>(tok) * r.k, r.w + static_cast<size_t>(tok) * r.k, hist);
      }
      // bounded sync of the 128 epilogue threads, then flush the histogram
      mbar_arrive(&epi_bar);
      if (mbar_wait(&epi_bar, 0, &abort_flag, r.status)) {
        for (int e = row; e < r.E; e += kRouteRows)
          if (hist[e]) atomicAdd(r.counts + e, hist[e]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, tmem_cols);
}

// ------------------------------------------------------------------------
// Kernel 2: routing from fp32 logits already in memory.
// ------------------------------------------------------------------------
__global__ void __launch_bounds__(kRouteRows)
route_logits_kernel(const RouteArgs r) {
  extern __shared__ __align__(16) float scratch_dyn[];
  __shared__ int hist[256];
  __shared__ float bias_s[256];
  const int row = threadIdx.x;
  const int tok = blockIdx.x * kRouteRows + row;
  for (int e = row; e < r.E; e += kRouteRows) {
    hist[e] = 0;
    bias_s[e] = r.bias ? r.bias[e] : 0.0f;
  }
  __syncthreads();
  float* col = scratch_dyn + row;
  float* gcol = scratch_dyn + static_cast<size_t>(kRouteRows) * r.E + row;
  const bool sig = r.scoring == MOE_SIGMOID;
  if (tok < r.T) {
    ScorePass sp;
    const float4* src = reinterpret_cast<const float4*>(r.logits + static_cast<size_t>(tok) * r.E);
    for (int c = 0; c * 32 < r.E; ++c) {
      float v[32];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float4 f = (c * 32 + 4 * j < r.E) ? src[c * 8 + j] : make_float4(0.f, 0.f, 0.f, 0.f);
        v[4 * j] = f.x; v[4 * j + 1] = f.y; v[4 * j + 2] = f.z; v[4 * j + 3] = f.w;
      }
      sp.chunk(col, v, c * 32, r.E, sig);
    }
    const double den = sig ? 1.0 : softmax_denominator(col, r.E, sp.lmax);
    route_token(col, gcol, r.bias ? bias_s : nullptr, sp.lmax, den, r,
                r.ids + static_cast<size_t>(tok) * r.k, r.w + static_cast<size_t>(tok) * r.k, hist);
  }
  __syncthreads();
  for (int e = row; e < r.E; e += kRouteRows)
    if (hist[e]) atomicAdd(r.counts + e, hist[e]);
}

// ------------------------------------------------------------------------
cudaError_t launch_route_gemm(const CUtensorMap& tmX, const CUtensorMap& tmG, const RouteArgs& r,
                              cudaStream_t stream) {
  uint32_t cols = 32;
  while (cols < static_cast<uint32_t>(r.E)) cols <<= 1;
  const size_t ring = static_cast<size_t>(kRouteStages) * (128 * 128 + static_cast<size_t>(r.E) * 128);
  const size_t scratch = route_scratch_bytes(r.E);
  const size_t smem = (ring > scratch ? ring : scratch) + 1024;
  cudaError_t e = cudaFuncSetAttribute(route_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int grid = (r.T + kRouteRows - 1) / kRouteRows;
  route_gemm_kernel<<<grid, 192, smem, stream>>>(tmX, tmG, r, cols);
  return cudaGetLastError();
}

cudaError_t launch_route_logits(const RouteArgs& r, cudaStream_t stream) {
  const size_t smem = route_scratch_bytes(r.E);
  cudaError_t e = cudaFuncSetAttribute(route_logits_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int grid = (r.T + kRouteRows - 1) / kRouteRows;
  route_logits_kernel<<<grid, kRouteRows, smem, stream>>>(r);
  return cudaGetLastError();
}

}  // namespace moe
