// Router: gate projection, scoring, group-limited top-k, routing weights.
//
// Pages: "MoE 混合专家模型推理参数与前向传播详解" §2.1 (router_logits =
// hidden_states @ gate.weight^T) and §3.1 (softmax scoring, greedy top-k, no
// renormalisation for V2-Lite); the gsyq.cn DeepSeek-V3 teardown §3-§4 (sigmoid
// scoring plus a balancing bias, n_group = 8 groups scored by the sum of their
// top-2, topk_group = 4 kept, top-8 within, renormalise, x routed_scaling_factor);
// the xxqk.cn digest §2.2 (bias only steers selection; device-limited routing).
//
// gate_route_kernel computes logits = x . gate^T on tcgen05: a cluster of
// SPLIT CTAs (2, 4 or 8; the most that still keeps every CTA of the grid
// resident at once) takes 128 tokens; CTA r accumulates over the r-th of SPLIT
// slices of the hidden size in its own TMEM (M = 128 tokens, N = E, fp32),
// then each CTA sends, through distributed shared memory, its partial sums of
// the 128/SPLIT tokens every other CTA owns. Every logit is the sum of the
// SPLIT partials in slice order. Where the shape allows (E = 8C with C in
// {2, 4, 8, 16, 32}, n_group | 8, k <= 8: every layer here) the same launch
// then routes the CTA's 128/SPLIT tokens from
// their logits in shared memory, eight threads per token, each holding E/8
// consecutive experts: groups are scored by the sum of their two best
// selection scores and ranked with shuffles, and the top-k is k rounds of
// an arg-max over the token's threads (larger score first, lower expert
// index on ties). route_tokens_g8_kernel does the same from logits in
// global memory (routing given logits); other shapes are routed by
// route_tokens_kernel, one warp per token, lane l holding experts l, l+32,
// ..., in the same decision order.

#include "kernels.cuh"

namespace moe {

constexpr int kRouteRows = 128;      // tokens per gate-GEMM tile
constexpr int kRouteStages = 4;
constexpr int kEpl = 8;              // experts per lane (E <= 256)
constexpr int kRouteWarps = 8;       // tokens in flight per routing CTA

// Score -> fp32 as the library states it: sigmoid in double, rounded once.
__device__ __forceinline__ float sigmoid_rn(float v) {
  return static_cast<float>(1.0 / (1.0 + exp(-static_cast<double>(v))));
}

// ------------------------------------------------------------------------
// Routing, one warp per token.
// ------------------------------------------------------------------------
// (ov, oe) beats (v, e): larger score, or equal score and lower expert index.
__device__ __forceinline__ bool beats(float v, int e, float ov, int oe) {
  return ov > v || (ov == v && oe < e);
}

__global__ void __launch_bounds__(kRouteWarps * 32)
route_tokens_kernel(const RouteArgs r) {
  __shared__ int hist[256];
  __shared__ float bias_s[256];
  __shared__ float sel_s[kRouteWarps][256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int e = threadIdx.x; e < r.E; e += blockDim.x) {
    hist[e] = 0;
    bias_s[e] = r.bias ? r.bias[e] : 0.0f;
  }
  __syncthreads();
  const bool sig = r.scoring == MOE_SIGMOID;
  const bool has_bias = r.bias != nullptr;
  const bool raw_logit = !sig && r.G == 1 && !has_bias;     // softmax, one group: select on logits
  const int gsz = r.E / r.G;
  float* my_sel = sel_s[warp];

  for (int tok = blockIdx.x * kRouteWarps + warp; tok < r.T; tok += gridDim.x * kRouteWarps) {
    const float* L = r.logits + static_cast<size_t>(tok) * r.E;
    float lg[kEpl], sel[kEpl], unb[kEpl];
    float lmax = -INFINITY;
#pragma unroll
    for (int i = 0; i < kEpl; ++i) {
      const int e = lane + 32 * i;
      lg[i] = e < r.E ? L[e] : -INFINITY;
      lmax = fmaxf(lmax, lg[i]);
    }
    double den = 1.0;
    if (!sig) {
#pragma unroll
      for (int d = 16; d > 0; d >>= 1) lmax = fmaxf(lmax, __shfl_xor_sync(0xffffffffu, lmax, d));
      double sum = 0.0;
#pragma unroll
      for (int i = 0; i < kEpl; ++i)
        if (lane + 32 * i < r.E) sum += exp(static_cast<double>(lg[i]) - static_cast<double>(lmax));
#pragma unroll
      for (int d = 16; d > 0; d >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, d);
      den = sum;
    }
#pragma unroll
    for (int i = 0; i < kEpl; ++i) {
      const int e = lane + 32 * i;
      if (e < r.E) {
        const float u = sig ? sigmoid_rn(lg[i])
                            : static_cast<float>(exp(static_cast<double>(lg[i]) - static_cast<double>(lmax)) / den);
        unb[i] = u;
        sel[i] = raw_logit ? lg[i] : (has_bias ? u + bias_s[e] : u);
      } else {
        unb[i] = 0.0f;
        sel[i] = -INFINITY;
      }
    }
    if (r.G > 1) {
      // group score = fp32 sum of the group's two largest selection scores
#pragma unroll
      for (int i = 0; i < kEpl; ++i)
        if (lane + 32 * i < r.E) my_sel[lane + 32 * i] = sel[i];
      __syncwarp();
      float gs = -INFINITY;
      if (lane < r.G) {
        float m1 = -INFINITY, m2 = -INFINITY;
        for (int e = lane * gsz; e < (lane + 1) * gsz; ++e) {
          const float v = my_sel[e];
          if (v > m1) { m2 = m1; m1 = v; } else if (v > m2) { m2 = v; }
        }
        gs = gsz >= 2 ? m1 + m2 : m1;
      }
      __syncwarp();
      // keep the topk_group best groups (lower group index first on ties)
      int rank_g = 0;
      for (int j = 0; j < r.G; ++j) {
        const float o = __shfl_sync(0xffffffffu, gs, j);
        rank_g += (o > gs || (o == gs && j < lane)) ? 1 : 0;
      }
      const uint32_t kept = __ballot_sync(0xffffffffu, lane < r.G && rank_g < r.g);
#pragma unroll
      for (int i = 0; i < kEpl; ++i) {
        const int e = lane + 32 * i;
        if (e < r.E && !((kept >> (e / gsz)) & 1u)) sel[i] = -INFINITY;
      }
    }
    // top-k: k rounds of a warp arg-max
    uint32_t taken = 0;
    int my_id = 0;
    float my_w = 0.0f;
    for (int j = 0; j < r.k; ++j) {
      float v = -INFINITY;
      int be = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < kEpl; ++i) {
        const int e = lane + 32 * i;
        if (e < r.E && !((taken >> i) & 1u) && beats(v, be, sel[i], e)) { v = sel[i]; be = e; }
      }
#pragma unroll
      for (int d = 16; d > 0; d >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, v, d);
        const int oe = __shfl_xor_sync(0xffffffffu, be, d);
        if (beats(v, be, ov, oe)) { v = ov; be = oe; }
      }
      const bool found = be < r.E;                     // false only when no score compares (NaN)
      const int owner = be & 31, slot = found ? be >> 5 : 0;
      float u = 0.0f;
#pragma unroll
      for (int i = 0; i < kEpl; ++i)
        if (i == slot) u = unb[i];
      u = __shfl_sync(0xffffffffu, u, owner);
      if (found && lane == owner) taken |= 1u << slot;
      if (lane == j) { my_id = found ? be : -1; my_w = found ? u : 0.0f; }
    }
    float sum = 0.0f;
    for (int j = 0; j < r.k; ++j) sum += __shfl_sync(0xffffffffu, my_w, j);
    if (lane < r.k) {
      const float w = (r.norm ? my_w / sum : my_w) * r.scale;
      r.ids[static_cast<size_t>(tok) * r.k + lane] = my_id;
      r.w[static_cast<size_t>(tok) * r.k + lane] = my_id >= 0 ? w : 0.0f;
      if (my_id >= 0) atomicAdd(&hist[my_id], 1);
      else flag_status(r.status, MOE_DEVSTAT_BAD_EXPERT_ID);
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < r.E; e += blockDim.x)
    if (hist[e]) atomicAdd(r.counts + e, hist[e]);
}

// ------------------------------------------------------------------------
// Routing, eight threads per token (E = 8C experts, C <= 32; n_group | 8;
// k <= 8): thread p of a token holds experts [pC, pC + C) in registers, so
// a group of E / n_group experts is whole threads and its top-2 merges over
// 8 / n_group threads by shuffles; the top-k is k rounds of an arg-max over
// the 8 threads; thread j < k writes slot j. The same decisions and weights
// as route_tokens_kernel (same scores, same order, same sums), in about half
// the instructions per token.
// ------------------------------------------------------------------------
// C consecutive scores from global or shared memory (generic loads).
template <int C>
__device__ __forceinline__ void load_scores(const float* src, float (&s)[C]) {
  if constexpr (C % 4 == 0) {
#pragma unroll
    for (int i = 0; i < C / 4; ++i) {
      const float4 v = reinterpret_cast<const float4*>(src)[i];
      s[4 * i] = v.x; s[4 * i + 1] = v.y; s[4 * i + 2] = v.z; s[4 * i + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < C / 2; ++i) {
      const float2 v = reinterpret_cast<const float2*>(src)[i];
      s[2 * i] = v.x; s[2 * i + 1] = v.y;
    }
  }
}

// Routes token `tok` (valid: tok < T) from its E logits at L, eight
// threads per token: lane bits 0..2 pick the thread's part (experts
// [pC, pC + C)), lane bits 3..4 the token of the warp's four. Every lane of
// the warp must call it (all lanes take part in every shuffle). Counts go to
// the shared histogram `hist`.
template <int C>
__device__ __forceinline__ void route_token8(const RouteArgs& r, const float* __restrict__ L, int tok, bool valid,
                                             const float* bias_s, int* hist) {
  constexpr uint32_t kAll = 0xffffffffu;
  const int lane = threadIdx.x & 31;
  const int p = lane & 7;                            // this thread's part of its token
  const int gl0 = lane & 24;                         // the token's first lane
  const bool sig = r.scoring == MOE_SIGMOID;
  const bool has_bias = r.bias != nullptr;
  const bool raw_logit = !sig && r.G == 1 && !has_bias;   // softmax, one group: select on logits
  const int tpg = 8 / r.G;                           // threads per group
  const int e0 = p * C;
  float s[C];
  load_scores<C>(L + e0, s);
  // softmax: max and denominator over the token's E logits
  float lmax = 0.0f;
  double den = 1.0;
  if (!sig) {
    lmax = -INFINITY;
#pragma unroll
    for (int i = 0; i < C; ++i) lmax = fmaxf(lmax, s[i]);
#pragma unroll
    for (int d = 1; d < 8; d <<= 1) lmax = fmaxf(lmax, __shfl_xor_sync(kAll, lmax, d));
    double sum = 0.0;
#pragma unroll
    for (int i = 0; i < C; ++i) sum += exp(static_cast<double>(s[i]) - static_cast<double>(lmax));
#pragma unroll
    for (int d = 1; d < 8; d <<= 1) sum += __shfl_xor_sync(kAll, sum, d);
    den = sum;
  }
  // selection scores, in place
  if (!raw_logit) {
#pragma unroll
    for (int i = 0; i < C; ++i) {
      const float u = sig ? sigmoid_rn(s[i])
                          : static_cast<float>(exp(static_cast<double>(s[i]) - static_cast<double>(lmax)) / den);
      s[i] = has_bias ? u + bias_s[e0 + i] : u;
    }
  }
  if (r.G > 1) {
    // group score = fp32 sum of the group's two largest selection scores
    float m1 = -INFINITY, m2 = -INFINITY;
#pragma unroll
    for (int i = 0; i < C; ++i) {
      const float v = s[i];
      if (v > m1) { m2 = m1; m1 = v; } else if (v > m2) { m2 = v; }
    }
    for (int d = 1; d < tpg; d <<= 1) {             // the two largest of both halves
      const float o1 = __shfl_xor_sync(kAll, m1, d), o2 = __shfl_xor_sync(kAll, m2, d);
      const float hi = fmaxf(m1, o1), lo = fminf(m1, o1);
      m2 = fmaxf(lo, fmaxf(m2, o2));
      m1 = hi;
    }
    const float gs = m1 + m2;
    // keep the topk_group best groups (lower group index first on ties)
    const int my_g = p / tpg;
    int rank_g = 0;
    for (int j = 0; j < r.G; ++j) {
      const float o = __shfl_sync(kAll, gs, gl0 + j * tpg);
      rank_g += (o > gs || (o == gs && j < my_g)) ? 1 : 0;
    }
    if (rank_g >= r.g) {
#pragma unroll
      for (int i = 0; i < C; ++i) s[i] = -INFINITY;
    }
  }
  // top-k: k rounds of an arg-max over the token's 8 threads
  uint32_t taken = 0;
  int my_id = 0;
  for (int j = 0; j < r.k; ++j) {
    float v = -INFINITY;
    int be = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < C; ++i)
      if (!((taken >> i) & 1u) && beats(v, be, s[i], e0 + i)) { v = s[i]; be = e0 + i; }
#pragma unroll
    for (int d = 1; d < 8; d <<= 1) {
      const float ov = __shfl_xor_sync(kAll, v, d);
      const int oe = __shfl_xor_sync(kAll, be, d);
      if (beats(v, be, ov, oe)) { v = ov; be = oe; }
    }
    const int rel = be - e0;
    if (rel >= 0 && rel < C) taken |= 1u << rel;
    if (p == j) my_id = be;
  }
  // weights: the unbiased score of slot p's expert, renormalised over the
  // k slots in slot order, times the scaling factor
  // (no expert wins a round only when no score compares, i.e. all are
  // NaN: the slot gets id -1, flagged, and counts nowhere)
  const bool has_id = my_id >= 0 && my_id < r.E;
  float u = 0.0f;
  if (p < r.k && valid && has_id) {
    const float lv = L[my_id];
    u = sig ? sigmoid_rn(lv) : static_cast<float>(exp(static_cast<double>(lv) - static_cast<double>(lmax)) / den);
  }
  float sum = 0.0f;
  for (int j = 0; j < r.k; ++j) sum += __shfl_sync(kAll, u, gl0 + j);
  if (p < r.k && valid) {
    const float w = (r.norm ? u / sum : u) * r.scale;
    r.ids[static_cast<size_t>(tok) * r.k + p] = has_id ? my_id : -1;
    r.w[static_cast<size_t>(tok) * r.k + p] = has_id ? w : 0.0f;
    if (has_id) atomicAdd(&hist[my_id], 1);
    else flag_status(r.status, MOE_DEVSTAT_BAD_EXPERT_ID);
  }
}

template <int C>
__global__ void __launch_bounds__(256, 2)
route_tokens_g8_kernel(const RouteArgs r) {
  __shared__ int hist[256];
  __shared__ float bias_s[256];
  for (int e = threadIdx.x; e < r.E; e += blockDim.x) {
    hist[e] = 0;
    bias_s[e] = r.bias ? r.bias[e] : 0.0f;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int nwarps = gridDim.x * (blockDim.x >> 5);
  // a warp routes four tokens per pass; every lane takes part in every shuffle
  for (int wq = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); wq * 4 < r.T; wq += nwarps) {
    const int tok = wq * 4 + (lane >> 3);
    const bool valid = tok < r.T;
    route_token8<C>(r, r.logits + static_cast<size_t>(valid ? tok : 0) * r.E, tok, valid, bias_s, hist);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < r.E; e += blockDim.x)
    if (hist[e]) atomicAdd(r.counts + e, hist[e]);
}

// ------------------------------------------------------------------------
// Gate GEMM on clusters of SPLIT CTAs, split along K, and (C > 0) the
// routing of the tile's tokens in the same launch.
// ------------------------------------------------------------------------
// 512 threads: warp 0 TMA producer, warp 1 TMEM allocator and MMA issuer,
// warps 2..5 read the accumulator (warp w: TMEM lanes 32*(w%4)..+31); after
// the exchange all sixteen warps route the CTA's 128/SPLIT tokens in one
// pass. The CTAs of a cluster start their K loop at a rotation that differs
// from cluster to cluster, so the clusters running side by side do not all
// read the same gate rows at the same moment (each CTA still sums its K
// blocks in one fixed order).
constexpr int kGateThreads = 512;

template <int C, int SPLIT>
__global__ void __launch_bounds__(kGateThreads, 1)
gate_route_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmG,
                  const RouteArgs r, uint32_t tmem_cols) {
  static_assert(SPLIT == 2 || SPLIT == 4 || SPLIT == 8, "clusters of 2, 4 or 8 CTAs");
  constexpr int KB = 64;
  constexpr int OWN = kRouteRows / SPLIT;              // tokens each CTA owns (and routes)
  extern __shared__ __align__(1024) uint8_t dsmem[];
  __shared__ uint64_t full_bar[kRouteStages], empty_bar[kRouteStages];
  __shared__ uint64_t tmem_full, drain_bar;
  __shared__ uint32_t tmem_base_s;
  __shared__ int issued_parity[kRouteStages];
  __shared__ volatile int abort_flag;
  __shared__ int hist[C > 0 ? 256 : 1];
  __shared__ float bias_s[C > 0 ? 256 : 1];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
  const uint32_t a_bytes = 128u * 128u;
  const uint32_t b_bytes = static_cast<uint32_t>(r.E) * 128u;
  const uint32_t stage_bytes = a_bytes + b_bytes;
  const int m0 = static_cast<int>(cluster_id_x()) * kRouteRows;
  const int nk = r.H / KB;
  // CTA r: the K blocks [r * nk / SPLIT, (r + 1) * nk / SPLIT)
  const int kb_begin = (static_cast<int>(rank) * nk) / SPLIT;
  const int kb_count = ((static_cast<int>(rank) + 1) * nk) / SPLIT - kb_begin;
  // after the main loop: recv[slot][OWN][LD], the other CTAs' partial sums of
  // this CTA's tokens (slot = the sender's rank with this CTA's left out);
  // rows padded by 16 bytes so that 32 rows' same column spread over the banks
  float* recv = reinterpret_cast<float*>(smem);
  const int LD = r.E + 4;
  const int rot = kb_count > 0 ? static_cast<int>((cluster_id_x() * 7u) % static_cast<uint32_t>(kb_count)) : 0;

  if constexpr (C > 0) {
    for (int e = threadIdx.x; e < r.E; e += blockDim.x) {
      hist[e] = 0;
      bias_s[e] = r.bias ? r.bias[e] : 0.0f;
    }
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < kRouteStages; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 1);
      issued_parity[i] = -1;
    }
    mbar_init(&tmem_full, 1);
    mbar_init(&drain_bar, 1);
    abort_flag = 0;
    fence_barrier_init();
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

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol_x = policy_evict_first();
      const uint64_t pol_g = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      for (int i = 0; i < kb_count; ++i) {
        const int kb = kb_begin + (i + rot < kb_count ? i + rot : i + rot - kb_count);
        if (!mbar_wait(&empty_bar[stage], phase ^ 1u, &abort_flag, r.status, r.wait_ns)) break;
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
      for (int i = 0; i < kb_count; ++i) {
        if (!mbar_wait(&full_bar[stage], phase, &abort_flag, r.status, r.wait_ns)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a0 = smem_u32(smem + stage * stage_bytes);
        const uint32_t b0 = a0 + a_bytes;
#pragma unroll
        for (int kk = 0; kk < KB / 16; ++kk)
          umma_bf16(tmem_base, sw128_desc(a0 + kk * 32), sw128_desc(b0 + kk * 32), idesc, (i | kk) != 0);
        umma_commit(&empty_bar[stage]);
        if (++stage == kRouteStages) { stage = 0; phase ^= 1u; }
      }
      if (ok && kb_count > 0) umma_commit(&tmem_full);
      umma_commit(&drain_bar);
      mbar_wait_drain(&drain_bar, 0);
    }
  } else if (kb_count > 0) {
    mbar_wait(&tmem_full, 0, &abort_flag, r.status, r.wait_ns);   // an abort still reaches the cluster barriers
    tc_fence_after();
  }
  // both CTAs: every MMA has completed (epilogue threads arrive only after
  // tmem_full), so the operand rings are free for the exchange
  cluster_sync();

  const int q = warp & 3;
  const int row = 32 * q + lane;                       // TMEM lane == token row of the tile
  const bool epi = warp >= 2 && warp < 6;
  const int owner = row / OWN;                         // CTA owner writes rows [OWN * owner, +OWN)
  const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(32 * q) << 16);
  // every lane of a warp reads the accumulator (tcgen05.ld is warp-collective)
  auto partial = [&](int c, float (&v)[32]) {
    if (kb_count > 0) {
      tmem_ld32(lane_addr + c * 32, v);
      tmem_ld_wait();
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = 0.0f;
    }
  };
  // a warp whose 32 rows are all this CTA's sends nothing; otherwise every
  // lane whose row another CTA owns sends it there
  const bool warp_all_mine = (32 * q) / OWN == static_cast<int>(rank) && (32 * q + 31) / OWN == static_cast<int>(rank);
  if (epi && !warp_all_mine) {
    const int slot = static_cast<int>(rank) < owner ? static_cast<int>(rank) : static_cast<int>(rank) - 1;
    const uint32_t dst = mapa_shared(smem_u32(recv), static_cast<uint32_t>(owner)) +
                         static_cast<uint32_t>((slot * OWN + row % OWN) * LD) * 4u;
    for (int c = 0; c * 32 < r.E; ++c) {
      float v[32];
      partial(c, v);
      if (owner != static_cast<int>(rank)) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (c * 32 + 4 * j < r.E)
            asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(dst + (c * 32 + 4 * j) * 4u),
                         "f"(v[4 * j]), "f"(v[4 * j + 1]), "f"(v[4 * j + 2]), "f"(v[4 * j + 3])
                         : "memory");
        }
      }
    }
  }
  cluster_sync();                                      // every partial has landed

  // this CTA's own rows [OWN * rank, +OWN): the warps holding them add the
  // SPLIT partial sums in rank order and write the logits (and, to route
  // them, keep them in slot 0 of recv)
  const bool warp_has_mine = (32 * q) / OWN <= static_cast<int>(rank) && static_cast<int>(rank) <= (32 * q + 31) / OWN;
  if (epi && warp_has_mine) {
    const bool mine = owner == static_cast<int>(rank);
    const int tok = m0 + row;
    const int i = row % OWN;
    for (int c = 0; c * 32 < r.E; ++c) {
      float v[32];
      partial(c, v);
      if (mine && tok < r.T) {
        float4* dst = reinterpret_cast<float4*>(r.logits + static_cast<size_t>(tok) * r.E + c * 32);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (c * 32 + 4 * j < r.E) {
            float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
            for (int src = 0; src < SPLIT; ++src) {           // partials added in rank order
              const int sl = src < static_cast<int>(rank) ? src : src - 1;
              const float4 pv = src == static_cast<int>(rank)
                                    ? make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3])
                                    : *reinterpret_cast<const float4*>(recv + (sl * OWN + i) * LD + c * 32 + 4 * j);
              if (src == 0) {
                acc = pv;
              } else {
                acc.x += pv.x; acc.y += pv.y; acc.z += pv.z; acc.w += pv.w;
              }
            }
            dst[j] = acc;
            if constexpr (C > 0) *reinterpret_cast<float4*>(recv + i * LD + c * 32 + 4 * j) = acc;
          }
        }
      }
    }
  }
  if constexpr (C > 0) {
    // route this CTA's OWN tokens from their logits in shared memory: each
    // warp four tokens (eight threads per token), all in one pass
    __syncthreads();
    const int tok_base = m0 + OWN * static_cast<int>(rank);
    const int i = 4 * warp + (lane >> 3);
    const int tok = tok_base + i;
    const bool valid = i < OWN && tok < r.T;
    route_token8<C>(r, recv + static_cast<size_t>(valid ? i : 0) * LD, tok, valid, bias_s, hist);
    __syncthreads();
    for (int e = threadIdx.x; e < r.E; e += blockDim.x)
      if (hist[e]) atomicAdd(r.counts + e, hist[e]);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, tmem_cols);
}

// ------------------------------------------------------------------------
int route8_experts_per_thread(const RouteArgs& r) {
  const int C = r.E / 8;
  const bool ok = r.E % 8 == 0 && r.k <= 8 && r.G >= 1 && 8 % r.G == 0 &&
                  (C == 2 || C == 4 || C == 8 || C == 16 || C == 32);
  return ok ? C : 0;
}

// Clusters of SPLIT CTAs per 128-token tile: the largest of 8, 4, 2 that still
// leaves every CTA resident at once (tiles * SPLIT <= the SM count), so few
// tokens still spread over many SMs while V3's 64 tiles keep pairs.
int gate_split(int T, int num_sms) {
  const int tiles = (T + kRouteRows - 1) / kRouteRows;
  for (int split = 8; split > 2; split >>= 1)
    if (tiles * split <= num_sms) return split;
  return 2;
}

template <int C, int SPLIT>
cudaError_t launch_gate_route_split(const CUtensorMap& tmX, const CUtensorMap& tmG, const RouteArgs& r,
                                    uint32_t cols, cudaStream_t stream) {
  const size_t ring = static_cast<size_t>(kRouteStages) * (128 * 128 + static_cast<size_t>(r.E) * 128);
  const size_t recv = static_cast<size_t>(SPLIT - 1) * (kRouteRows / SPLIT) * (r.E + 4) * sizeof(float);
  const size_t smem = (ring > recv ? ring : recv) + 1024;
  auto kern = gate_route_kernel<C, SPLIT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(SPLIT * ((r.T + kRouteRows - 1) / kRouteRows));
  cfg.blockDim = dim3(kGateThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = SPLIT;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, tmX, tmG, r, cols);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int C>
cudaError_t launch_gate_route(const CUtensorMap& tmX, const CUtensorMap& tmG, const RouteArgs& r, uint32_t cols,
                              int split, cudaStream_t stream) {
  if (split == 8) return launch_gate_route_split<C, 8>(tmX, tmG, r, cols, stream);
  if (split == 4) return launch_gate_route_split<C, 4>(tmX, tmG, r, cols, stream);
  return launch_gate_route_split<C, 2>(tmX, tmG, r, cols, stream);
}

cudaError_t launch_gate_gemm(const CUtensorMap& tmX, const CUtensorMap& tmG, const RouteArgs& r, bool route,
                             int num_sms, cudaStream_t stream) {
  uint32_t cols = 32;
  while (cols < static_cast<uint32_t>(r.E)) cols <<= 1;
  const int split = gate_split(r.T, num_sms);
  switch (route ? route8_experts_per_thread(r) : 0) {
    case 2: return launch_gate_route<2>(tmX, tmG, r, cols, split, stream);
    case 4: return launch_gate_route<4>(tmX, tmG, r, cols, split, stream);
    case 8: return launch_gate_route<8>(tmX, tmG, r, cols, split, stream);
    case 16: return launch_gate_route<16>(tmX, tmG, r, cols, split, stream);
    case 32: return launch_gate_route<32>(tmX, tmG, r, cols, split, stream);
    default: return launch_gate_route<0>(tmX, tmG, r, cols, split, stream);
  }
}

cudaError_t launch_route_tokens(const RouteArgs& r, int num_sms, cudaStream_t stream) {
  // eight threads per token where the shape allows, else one warp per token
  const int C = route8_experts_per_thread(r);
  if (C > 0) {
    const int need = (r.T + 31) / 32;                 // 32 tokens per CTA of 256 threads
    const int grid = need < 4 * num_sms ? need : 4 * num_sms;
    switch (C) {
      case 2: route_tokens_g8_kernel<2><<<grid, 256, 0, stream>>>(r); break;
      case 4: route_tokens_g8_kernel<4><<<grid, 256, 0, stream>>>(r); break;
      case 8: route_tokens_g8_kernel<8><<<grid, 256, 0, stream>>>(r); break;
      case 16: route_tokens_g8_kernel<16><<<grid, 256, 0, stream>>>(r); break;
      default: route_tokens_g8_kernel<32><<<grid, 256, 0, stream>>>(r); break;
    }
    return cudaGetLastError();
  }
  const int need = (r.T + kRouteWarps - 1) / kRouteWarps;
  const int grid = need < 8 * num_sms ? need : 8 * num_sms;
  route_tokens_kernel<<<grid, kRouteWarps * 32, 0, stream>>>(r);
  return cudaGetLastError();
}

}  // namespace moe
