// Grouped SwiGLU expert GEMMs on the 5th-generation tensor cores (tcgen05).
//
// The layer's experts ("MoE 混合专家模型推理参数与前向传播详解" §3.3.1):
//   gate_up = x @ w13[e]^T ; h = SiLU(gate_up[:, :I]) * gate_up[:, I:]
//   out     = h @ w2[e]^T  (times the row's routing weight, §3.4)
// run for every expert in one launch over the expert-contiguous rows produced
// by the permutation (§3.2), i.e. a grouped GEMM segmented by expert offsets.
//
// Orientation (swap-AB): the weight matrix is the MMA's A operand (M = 128
// weight rows per tcgen05.mma) and the segment's token rows are the B operand
// (N = 16..256 tokens, variable per tile). A segment of n rows costs
// round_up(n, 16) columns, so ragged segment ends waste at most 15 columns,
// instead of most of a 128-row tile when tokens sit on the M side.
//
// Tile = (expert g, weight block mb, token block tb), rasterised per segment
// in chunks of token blocks (token block innermost). Each tile holds two
// 128-row sub-tiles of the weight, accumulated side by side in TMEM:
//   GEMM1: sub-tile 0 = gate rows [mb*128, +128), sub-tile 1 = up rows
//          [I + mb*128, +128): the epilogue has gate and up of the same
//          feature in the same thread and fuses SiLU(gate) * up.
//   GEMM2: sub-tiles = w2 rows [mb*256, +128) and [mb*256 + 128, +128); the
//          epilogue multiplies by the routing weight of the row.
// TMEM (512 fp32 columns) holds one accumulator pair of up to 256 tokens.
// 256-token tiles read each 3.7 MB weight tile (V3 gate/up) half as often as
// 128-token tiles would, which at the V3 shape on B200 was measured to be
// worth more than double-buffering the accumulator (which would halve the
// tile) to overlap the epilogue with the next tile's MMAs.
//
// Warp roles (one CTA per SM, persistent over tiles):
//   warp 0      TMA producer (A: the weight rows, B: the tile's token rows in
//               boxes of 256/128/64/32/16 rows, 128-byte swizzle) into a ring
//               of three 64-K stages;
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer;
//   warps 2..   epilogue (4 warps for GEMM1, 12 for GEMM2, whose output is
//               twice as wide): tcgen05.ld (warp w reads TMEM lanes
//               32*(w%4)..+31), fused activation / weighting, bf16 stores.
// A launch may carry a second, single-group problem (the shared expert) whose
// tiles come first in the tile order.
// The E4M3 variant accumulates each 128-wide K block separately in a TMEM
// ring and promotes it with the fp32 block scales on the CUDA cores, since
// the weight scale is per 128x128 block and the activation scale per 1x128.
#include "kernels.cuh"

namespace moe {

constexpr int kMaxGroups = 512;
constexpr int kThreads = 192;

struct TileInfo {
  int g, mb, row0, n_valid, N;
  int ntb;              // token blocks of this segment
  int tb;               // this tile's token block in the segment
};

// Token blocks per rasterisation chunk: inside a segment, tiles run in chunks
// of up to kTbChunk token blocks x all weight blocks, token block innermost,
// so CTAs running side by side share the weight block (HBM once, then L2)
// and the chunk's token blocks (L2).
constexpr int kTbChunk = 8;

// Pipeline stages of 64 K: bf16 (64 KB each), E4M3.
constexpr int kBf16Stages = 3;
constexpr int kE4m3Stages = 4;

// Per-CTA copy of the tile schedule: tb_start[g] = first token block of
// group g (over all groups), tile_start[g] = its first tile (tb_start[g] x
// the problem's weight blocks).
struct Sched {
  int tile_start[kMaxGroups + 1];
  int seg_start[kMaxGroups + 1];
  int tb_start[kMaxGroups + 1];
};

__device__ __forceinline__ int tiles_of(int n, int bn_max, int n_mblk) {
  return n <= 0 ? 0 : ((n + bn_max - 1) / bn_max) * n_mblk;
}

// Warp-cooperative build of the schedule (called by one warp).
__device__ void build_schedule(Sched& s, const GemmArgs& a, int lane) {
  int carry = 0;
  for (int base = 0; base < a.groups; base += 32) {
    const int g = base + lane;
    int st = 0, n = 0;
    if (g < a.groups) {
      if (a.offsets) {
        st = a.offsets[g];
        n = a.offsets[g + 1] - st;
      } else {
        st = 0;
        n = a.rows;
      }
    }
    int t = (g < a.groups) ? tiles_of(n, a.bn_max, 1) : 0;   // token blocks
    int incl = t;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      int v = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += v;
    }
    if (g < a.groups) {
      s.tb_start[g] = carry + incl - t;
      s.tile_start[g] = (carry + incl - t) * a.n_mblk;
      s.seg_start[g] = st;
    }
    carry += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) {
    s.tb_start[a.groups] = carry;
    s.tile_start[a.groups] = carry * a.n_mblk;
    s.seg_start[a.groups] = a.offsets ? a.offsets[a.groups] : a.rows;
  }
}

// Tile `local` of a segment of n rows starting at row seg0 (group g).
__device__ __forceinline__ TileInfo decode_in_segment(const GemmArgs& a, int g, int seg0, int n, int local) {
  TileInfo ti;
  ti.g = g;
  const int ntb = (n + a.bn_max - 1) / a.bn_max;
  const int bn = ((((n + ntb - 1) / ntb) + 15) / 16) * 16;
  const int chunk_tiles = kTbChunk * a.n_mblk;
  const int chunk = local / chunk_tiles;
  const int r = local - chunk * chunk_tiles;
  const int c_tb = min(kTbChunk, ntb - chunk * kTbChunk);   // token blocks in this chunk
  ti.mb = r / c_tb;
  const int tb = chunk * kTbChunk + (r - ti.mb * c_tb);
  ti.ntb = ntb;
  ti.tb = tb;
  ti.row0 = seg0 + tb * bn;
  ti.n_valid = min(bn, n - tb * bn);
  ti.N = ((ti.n_valid + 15) / 16) * 16;
  return ti;
}

__device__ __forceinline__ TileInfo decode_tile(const Sched& s, const GemmArgs& a, int t) {
  int lo = 0, hi = a.groups - 1;   // last g with tile_start[g] <= t
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (s.tile_start[mid] <= t) lo = mid; else hi = mid - 1;
  }
  return decode_in_segment(a, lo, s.seg_start[lo], s.seg_start[lo + 1] - s.seg_start[lo],
                           t - s.tile_start[lo]);
}

// Tile t of problem a over the schedule's segments when a's weight blocks per
// group differ from those the schedule was built with (its token blocks are
// the same: same offsets and bn_max).
__device__ __forceinline__ TileInfo decode_tile_nb(const Sched& s, const GemmArgs& a, int t) {
  int lo = 0, hi = a.groups - 1;   // last g with tb_start[g] * n_mblk <= t
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (s.tb_start[mid] * a.n_mblk <= t) lo = mid; else hi = mid - 1;
  }
  return decode_in_segment(a, lo, s.seg_start[lo], s.seg_start[lo + 1] - s.seg_start[lo],
                           t - s.tb_start[lo] * a.n_mblk);
}

// The weight rows of K block kb of a tile. Row-major weights: sub-tiles at
// rows a_row0 and a_row1 (128 rows each), or one 256-row box at a_row0, read
// at (kb * 64, row). Tiled weights (moe_tile_ffn_weights, wblk >= 0): the
// tile's 256 rows of K block kb (gate/up: the 128 gate rows, then the 128 up
// rows) are one contiguous block at row (wblk * nk + kb) * 256.
__device__ __forceinline__ void load_weight_rows(void* dst0, void* dst1, const CUtensorMap* mA, uint64_t* bar,
                                                 int kb, int nk, int a_row0, int a_row1, bool one_box, int wblk,
                                                 uint64_t pol) {
  constexpr int KB = 64;
  if (wblk >= 0) {
    tma_load_2d(dst0, mA, bar, 0, (wblk * nk + kb) * 256, pol);
  } else {
    tma_load_2d(dst0, mA, bar, kb * KB, a_row0, pol);
    if (!one_box) tma_load_2d(dst1, mA, bar, kb * KB, a_row1, pol);
  }
}

// Token rows of one stage (a multiple of 16, at most 256) are fetched with at
// most one box of each size 256, 128, 64, 32, 16: the binary digits of
// rows / 16. Returns rows loaded.
template <typename LoadFn>
__device__ __forceinline__ int load_token_rows(int rows, LoadFn&& load) {
  int off = 0;
#pragma unroll
  for (int i = 0; i < kTokBoxes; ++i) {
    const int box = 256 >> i;
    if (rows - off >= box) { load(i, off); off += box; }
  }
  return off;
}

// Writes NT tokens x 32 features (thread = feature lane, v[j] = token j) to
// out[(row0 + j) * ld + feat0 + lane] through a per-warp shared tile, so that
// every global store is a 16-byte vector (4 lanes cover one token's 32
// features). Tokens j >= n_rows are not written.
template <int NT>
__device__ __forceinline__ void store_tile(__nv_bfloat16* stage, const float (&v)[NT], int lane,
                                           __nv_bfloat16* out, size_t ld, int row0, int n_rows, int feat0) {
#pragma unroll
  for (int j = 0; j < NT; ++j) stage[j * 32 + lane] = __float2bfloat16_rn(v[j]);
  __syncwarp();
#pragma unroll
  for (int i = 0; i < NT / 8; ++i) {
    const int t = (lane >> 2) + 8 * i;
    const int seg = lane & 3;
    if (t < n_rows) {
      const uint4 val = *reinterpret_cast<const uint4*>(stage + t * 32 + seg * 8);
      *reinterpret_cast<uint4*>(out + static_cast<size_t>(row0 + t) * ld + feat0 + seg * 8) = val;
    }
  }
  __syncwarp();
}

// SiLU(g) = g * sigmoid(g). Fast division: for g < -88 the exponential
// overflows to inf and the quotient is the correct limit (-0).
__device__ __forceinline__ float silu(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

// ========================================================================
// BF16 kernel
// ========================================================================
// GATHER: two more warps (6, 7) fetch the token rows of every stage from
// a.gather_src at rows a.gather_rows[p] with 16-byte cp.async, writing the
// same 128-byte-swizzled layout TMA would (16-byte chunk c of row r lands at
// r * 128 + (c ^ (r % 8)) * 16). Each gather thread arrives on a stage's full
// barrier once its copies of that stage have landed and been fenced to the
// async proxy; it keeps one stage of copies in flight ahead of that.
constexpr int kGatherThreads = 64;


// TWO: a second single-group problem a2 (the shared expert: its own weights
// tmA2, token rows tmB2 and output) runs in the same launch. Its tiles come
// first in the tile order, so the routed experts' ragged tiles fill the tail.
template <int EPI, int STAGES, bool GATHER, bool TWO, int EPIW = 4>
__global__ void __launch_bounds__(64 + 32 * EPIW + (GATHER ? kGatherThreads : 0), 1)
grouped_gemm_bf16_kernel(const __grid_constant__ CUtensorMap tmA,
                         const __grid_constant__ TokenMaps tmB, const GemmArgs a,
                         const __grid_constant__ CUtensorMap tmA2,
                         const __grid_constant__ TokenMaps tmB2, const GemmArgs a2) {
  constexpr int KB = 64;                           // K elements per stage (128 B)
  constexpr uint32_t A_SUB_BYTES = 128 * 128;      // one 128-row sub-tile
  extern __shared__ __align__(1024) uint8_t dsmem[];
  __shared__ Sched sched;
  __shared__ __align__(16) __nv_bfloat16 stage_out[EPIW][32 * 32];
  __shared__ uint64_t full_bar[STAGES], empty_bar[STAGES];
  __shared__ uint64_t tmem_full, tmem_empty, drain_bar;
  __shared__ uint32_t tmem_base_s;
  __shared__ int issued_parity[STAGES];
  __shared__ volatile int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
  const uint32_t b_stage_bytes = static_cast<uint32_t>(a.bn_max) * 128u;
  // TMEM: one accumulator pair, sub-tile s in columns [s * 256, +256)
  constexpr uint32_t sub_cols = 256u;
  const uint64_t wait_ns = a.wait_ns;
  // a stage holds 64 K: [A sub-tile 0][A sub-tile 1][B rows]
  const uint32_t stage_bytes = 2 * A_SUB_BYTES + b_stage_bytes;
  auto sA = [&](int st, int sub) { return smem + st * stage_bytes + sub * A_SUB_BYTES; };
  auto sB = [&](int st) { return smem + st * stage_bytes + 2 * A_SUB_BYTES; };

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full_bar[i], GATHER ? 1 + kGatherThreads : 1);
      mbar_init(&empty_bar[i], 1);
      issued_parity[i] = -1;
    }
    mbar_init(&tmem_full, 1);
    mbar_init(&tmem_empty, 32 * EPIW);
    mbar_init(&drain_bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    for (int i = 0; i < kTokBoxes; ++i) tma_prefetch_desc(&tmB.box[i]);
    if (TWO) {
      tma_prefetch_desc(&tmA2);
      for (int i = 0; i < kTokBoxes; ++i) tma_prefetch_desc(&tmB2.box[i]);
    }
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_s, 512);
    tmem_relinquish();
  }
  if (warp == 2) build_schedule(sched, a, lane);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_s;
  const int total2 = TWO ? tiles_of(a2.rows, a.bn_max, a2.n_mblk) : 0;
  const int total = total2 + sched.tile_start[a.groups];

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol_once = policy_evict_first();
      const uint64_t pol_reuse = policy_evict_normal();
      const uint64_t pol_x = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      for (int t = blockIdx.x; t < total && !abort_flag; t += gridDim.x) {
        const bool sh = TWO && t < total2;
        const TileInfo ti = sh ? decode_in_segment(a2, 0, 0, a2.rows, t) : decode_tile(sched, a, t - total2);
        const int nk = (sh ? a2.K : a.K) / KB;
        const CUtensorMap* mA = sh ? &tmA2 : &tmA;
        const TokenMaps* mB = sh ? &tmB2 : &tmB;
        const int a_row0 = sh ? ti.mb * a2.mblk_stride : ti.g * a.a_rows_per_group + ti.mb * a.mblk_stride;
        const int a_row1 = a_row0 + (sh ? a2.sub1_off : a.sub1_off);
        const bool one_box = sh ? a2.a_one_box != 0 : a.a_one_box != 0;
        const int wblk = !(sh ? a2.a_tiled : a.a_tiled) ? -1 : sh ? ti.mb : ti.g * a.n_mblk + ti.mb;
        const uint64_t pol_w = ti.ntb > 1 ? pol_reuse : pol_once;   // re-read by sibling token blocks
        const uint32_t bytes = 2 * A_SUB_BYTES + (GATHER ? 0u : static_cast<uint32_t>(ti.N) * 128u);
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u, &abort_flag, a.status, wait_ns)) { ok = false; break; }
          mbar_arrive_expect_tx(&full_bar[stage], bytes);
          load_weight_rows(sA(stage, 0), sA(stage, 1), mA, &full_bar[stage], kb, nk, a_row0, a_row1, one_box, wblk,
                           pol_w);
          if (!GATHER) {
            uint8_t* bdst = sB(stage);
            uint64_t* fb = &full_bar[stage];
            load_token_rows(ti.N, [&](int which, int off) {
              tma_load_2d(bdst + off * 128, &mB->box[which], fb, kb * KB, ti.row0 + off, pol_x);
            });
          }
          issued_parity[stage] = static_cast<int>(phase);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
      }
      if (abort_flag) {   // let every issued copy land before the CTA exits
        for (int i = 0; i < STAGES; ++i)
          if (issued_parity[i] >= 0) mbar_wait_drain(&full_bar[i], static_cast<uint32_t>(issued_parity[i]));
      }
    }
  } else if (GATHER && warp >= 2 + EPIW) {
    const int gt = threadIdx.x - (64 + 32 * EPIW);    // 0..63
    const int chunk = gt & 7;                          // 16-byte chunk of the 128-byte row slice
    const __nv_bfloat16* src = reinterpret_cast<const __nv_bfloat16*>(a.gather_src);
    const int nk = a.K / KB;                          // (no second problem with GATHER)
    int stage = 0, pending = -1;
    uint32_t phase = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok && !abort_flag; t += gridDim.x) {
      const TileInfo ti = decode_tile(sched, a, t);
      int srow[32];                                    // source rows of this thread's token rows
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int r = (gt >> 3) + 8 * i;
        int sr = (r < ti.n_valid) ? __ldg(a.gather_rows + ti.row0 + r) : -1;
        if (sr >= a.gather_src_rows) { flag_status(a.status, MOE_DEVSTAT_BAD_EXPERT_ID); sr = -1; }
        srow[i] = sr;
      }
      for (int kb = 0; kb < nk; ++kb) {
        if (!mbar_wait(&empty_bar[stage], phase ^ 1u, &abort_flag, a.status, wait_ns)) { ok = false; break; }
        const uint32_t bbase = smem_u32(sB(stage));
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int r = (gt >> 3) + 8 * i;
          if (srow[i] >= 0)
            cp_async_16(bbase + r * 128 + ((chunk ^ (r & 7)) << 4),
                        src + static_cast<size_t>(srow[i]) * a.K + kb * KB + chunk * 8);
        }
        cp_async_commit();
        if (pending >= 0) {                            // the previous stage has landed
          cp_async_wait<1>();
          fence_proxy_async();
          mbar_arrive(&full_bar[pending]);
        }
        pending = stage;
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
    }
    cp_async_wait<0>();
    if (pending >= 0 && ok) {
      fence_proxy_async();
      mbar_arrive(&full_bar[pending]);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, it = 0;
      for (int t = blockIdx.x; t < total && !abort_flag; t += gridDim.x, ++it) {
        const bool sh = TWO && t < total2;
        const TileInfo ti = sh ? decode_in_segment(a2, 0, 0, a2.rows, t) : decode_tile(sched, a, t - total2);
        const int nk = (sh ? a2.K : a.K) / KB;
        const uint32_t idesc = make_idesc(1u, 128u, static_cast<uint32_t>(ti.N));
        const uint32_t d0 = tmem_base;
        if (!mbar_wait(&tmem_empty, (it & 1u) ^ 1u, &abort_flag, a.status, wait_ns)) break;
        tc_fence_after();
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase, &abort_flag, a.status, wait_ns)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA(stage, 0)), a1 = smem_u32(sA(stage, 1));
          const uint32_t b0 = smem_u32(sB(stage));
#pragma unroll
          for (int kk = 0; kk < KB / 16; ++kk) {
            const uint32_t acc = (kb | kk) != 0;
            const uint64_t bd = sw128_desc(b0 + kk * 32);
            umma_bf16(d0, sw128_desc(a0 + kk * 32), bd, idesc, acc);
            umma_bf16(d0 + sub_cols, sw128_desc(a1 + kk * 32), bd, idesc, acc);
          }
          umma_commit(&empty_bar[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(&tmem_full);
      }
      // all issued MMAs must finish before TMEM is released
      umma_commit(&drain_bar);
      mbar_wait_drain(&drain_bar, 0);
    }
  } else if (warp < 2 + EPIW) {
    // epilogue warps 2 .. 1+EPIW: warp w reads TMEM lanes 32*(w%4)..+31; with
    // 8 or 12 warps, two or three share each lane quarter and take turns on
    // its 32-token chunks
    const int q = warp & 3;
    const int c0 = (warp - 2) / 4, cstep = EPIW / 4;
    const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(32 * q) << 16);
    uint32_t it = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++it) {
      const bool sh = TWO && t < total2;
      const TileInfo ti = sh ? decode_in_segment(a2, 0, 0, a2.rows, t) : decode_tile(sched, a, t - total2);
      __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(sh ? a2.out : a.out);
      const size_t out_ld = sh ? a2.out_ld : a.out_ld;
      const int feat_stride = sh ? a2.feat_stride : a.feat_stride;
      const int feat_sub1 = sh ? a2.feat_sub1 : a.feat_sub1;
      const float* row_w = sh ? a2.row_w : a.row_w;
      const int nchunk = (ti.N + 31) / 32;
      // GEMM2: the routing weights (and, for the scatter, the tokens) of this
      // warp's 32-row chunks, fetched before the accumulator is ready so that
      // their latency overlaps the wait instead of each chunk's epilogue
      // 32-row chunks of a tile (at most 8) an epilogue warp handles at most
      constexpr int kEpiChunks = (8 + EPIW / 4 - 1) / (EPIW / 4);
      float wpre[kEpiChunks];
      int tpre[kEpiChunks];
      if (EPI != EPI_SWIGLU) {
        const int32_t* src = sh ? a2.scatter_tok : a.scatter_tok;
        const int ntok = sh ? a2.scatter_T : a.scatter_T;
#pragma unroll
        for (int u = 0; u < kEpiChunks; ++u) {
          const int r = (c0 + u * cstep) * 32 + lane;            // row within the tile
          const bool valid = c0 + u * cstep < nchunk && r < ti.n_valid;
          wpre[u] = (row_w && valid) ? __ldg(row_w + ti.row0 + r) : 0.0f;
          int tok = -1;
          if (EPI == EPI_SCATTER && valid) {
            tok = src ? __ldg(src + ti.row0 + r) : ti.row0 + r;   // routed rows through src_token
            if (tok >= ntok) { flag_status(a.status, MOE_DEVSTAT_BAD_EXPERT_ID); tok = -1; }
          }
          tpre[u] = tok;
        }
      }
      if (!mbar_wait(&tmem_full, it & 1u, &abort_flag, a.status, wait_ns)) break;
      tc_fence_after();
      const uint32_t acc_addr = lane_addr;
      __nv_bfloat16* stg = stage_out[warp - 2];
      if (EPI == EPI_SWIGLU) {
        const int feat0 = ti.mb * feat_stride + 32 * q;            // this warp's 32 features
        for (int c = c0; c < nchunk; c += cstep) {
          float g[32], u[32];
          tmem_ld32(acc_addr + c * 32, g);
          tmem_ld32(acc_addr + sub_cols + c * 32, u);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) g[j] = silu(g[j]) * u[j];
          store_tile<32>(stg, g, lane, out, out_ld, ti.row0 + c * 32, ti.n_valid - c * 32, feat0);
        }
      } else {
#pragma unroll 1
        for (int s = 0; s < 2; ++s) {
          const int feat0 = ti.mb * feat_stride + s * feat_sub1 + 32 * q;
#pragma unroll
          for (int u = 0; u < kEpiChunks; ++u) {
            const int c = c0 + u * cstep;
            if (c >= nchunk) break;                                  // warp-uniform
            float v[32];
            tmem_ld32(acc_addr + s * sub_cols + c * 32, v);
            tmem_ld_wait();
            if (row_w) {
#pragma unroll
              for (int j = 0; j < 32; ++j) v[j] *= __shfl_sync(0xffffffffu, wpre[u], j);
            }
            if (EPI == EPI_SCATTER) {
              float* acc_out = reinterpret_cast<float*>(sh ? a2.out : a.out);
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                const int tj = __shfl_sync(0xffffffffu, tpre[u], j);
                if (tj >= 0) atomicAdd(acc_out + static_cast<size_t>(tj) * out_ld + feat0 + lane, v[j]);
              }
            } else {
              store_tile<32>(stg, v, lane, out, out_ld, ti.row0 + c * 32, ti.n_valid - c * 32, feat0);
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tmem_empty);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, 512);
}

// ========================================================================
// Both GEMMs of the SwiGLU experts in one persistent launch (bf16)
// ========================================================================
// Tiles in order: shared gate/up, routed gate/up, shared down, routed down,
// each problem rasterised as in the kernel above, all on 256-token tiles with
// one accumulator pair and 12 epilogue warps. The CTAs take tiles from a
// global counter, in order, so the work is shared out to the end (a CTA
// whose tiles ran fast takes more) and the down tiles start on the SMs that
// finish their gate/up share first. A down tile reads the h rows of one
// token block: the gate/up epilogue warps, after storing their part of a
// tile, fence and add 1 to that token block's counter, and the down tile's
// producer waits (bounded) for n_mblk(gate/up) x 4 x kGuQ arrivals, then
// fences the async proxy before its TMA loads of those rows. Tiles are
// handed out in increasing order and a producer only waits after issuing
// every load of its earlier tiles, so each awaited gate/up tile completes.
// The tile a stage holds travels with the stage (stage_tile), the tile in
// the accumulator from the MMA warp to the epilogue warps (acc_tile,
// tile_bar); -1 marks the end.
__global__ void __launch_bounds__(64 + 32 * kFfnEpiWarps, 1)
grouped_ffn_bf16_kernel(const __grid_constant__ FfnArgs f) {
  constexpr int EPIW = kFfnEpiWarps;
  constexpr int STAGES = kBf16Stages;
  constexpr int KB = 64;
  constexpr uint32_t A_SUB_BYTES = 128 * 128;
  constexpr uint32_t sub_cols = 256u;
  extern __shared__ __align__(1024) uint8_t dsmem[];
  __shared__ Sched sched;
  __shared__ __align__(16) __nv_bfloat16 stage_out[EPIW][32 * 32];
  __shared__ uint64_t full_bar[STAGES], empty_bar[STAGES];
  __shared__ uint64_t tmem_full, tmem_empty, drain_bar, tile_bar;
  __shared__ uint32_t tmem_base_s;
  __shared__ int issued_parity[STAGES];
  __shared__ int stage_tile[STAGES];
  __shared__ int acc_tile;
  __shared__ volatile int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const GemmArgs& gr = f.g[1];                       // routed gate/up: the schedule's segments
  int32_t* status = gr.status;
  const uint64_t wait_ns = gr.wait_ns;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
  const uint32_t stage_bytes = 2 * A_SUB_BYTES + static_cast<uint32_t>(gr.bn_max) * 128u;
  auto sA = [&](int st, int sub) { return smem + st * stage_bytes + sub * A_SUB_BYTES; };
  auto sB = [&](int st) { return smem + st * stage_bytes + 2 * A_SUB_BYTES; };

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 1);
      issued_parity[i] = -1;
    }
    mbar_init(&tmem_full, 1);
    mbar_init(&tmem_empty, 32 * EPIW);
    mbar_init(&drain_bar, 1);
    mbar_init(&tile_bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    for (int p = 0; p < 4; ++p) {
      tma_prefetch_desc(&f.tmA[p]);
      for (int i = 0; i < kTokBoxes; ++i) tma_prefetch_desc(&f.tmB[p].box[i]);
    }
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_s, 512);
    tmem_relinquish();
  }
  if (warp == 2) build_schedule(sched, gr, lane);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_s;
  const int tb_routed = sched.tb_start[gr.groups];
  // first tile of problems 1, 2, 3, and the total
  const int first1 = tiles_of(f.g[0].rows, f.g[0].bn_max, f.g[0].n_mblk);
  const int first2 = first1 + tb_routed * f.g[1].n_mblk;
  const int first3 = first2 + tiles_of(f.g[2].rows, f.g[2].bn_max, f.g[2].n_mblk);
  const int total = first3 + tb_routed * f.g[3].n_mblk;
  // problem of tile t, its tile info and its token block's counter
  auto locate = [&](int t, int& p, TileInfo& ti) -> int {
    p = t < first1 ? 0 : t < first2 ? 1 : t < first3 ? 2 : 3;
    const int base = p == 0 ? 0 : p == 1 ? first1 : p == 2 ? first2 : first3;
    const GemmArgs& g = f.g[p];
    if (p == 0 || p == 2) {
      ti = decode_in_segment(g, 0, 0, g.rows, t - base);
      return f.shared_base + ti.tb;
    }
    ti = decode_tile_nb(sched, g, t - base);
    return sched.tb_start[ti.g] + ti.tb;
  };

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol_once = policy_evict_first();
      const uint64_t pol_reuse = policy_evict_normal();
      const uint64_t pol_x = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      int next = atomicAdd(f.tile_counter, 1);
      while (next < total && !abort_flag) {
        const int t = next;
        int p;
        TileInfo ti;
        const int idx = locate(t, p, ti);
        const GemmArgs& g = f.g[p];
        if (p >= 2) {                                  // h rows of this token block stored and visible
          const int32_t target = f.g[p - 2].n_mblk * 4 * kGuQ;
          if (!wait_count(f.ready + idx, target, &abort_flag, status, wait_ns)) break;
          fence_proxy_async_global();
        }
        const int nk = g.K / KB;
        const CUtensorMap* mA = &f.tmA[p];
        const TokenMaps* mB = &f.tmB[p];
        const int a_row0 = ti.g * g.a_rows_per_group + ti.mb * g.mblk_stride;
        const int a_row1 = a_row0 + g.sub1_off;
        const bool one_box = g.a_one_box != 0;
        const int wblk = g.a_tiled ? ti.g * g.n_mblk + ti.mb : -1;
        const uint64_t pol_w = ti.ntb > 1 ? pol_reuse : pol_once;
        const uint32_t bytes = 2 * A_SUB_BYTES + static_cast<uint32_t>(ti.N) * 128u;
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u, &abort_flag, status, wait_ns)) { ok = false; break; }
          stage_tile[stage] = t;
          mbar_arrive_expect_tx(&full_bar[stage], bytes);
          load_weight_rows(sA(stage, 0), sA(stage, 1), mA, &full_bar[stage], kb, nk, a_row0, a_row1, one_box, wblk,
                           pol_w);
          uint8_t* bdst = sB(stage);
          uint64_t* fb = &full_bar[stage];
          load_token_rows(ti.N, [&](int which, int off) {
            tma_load_2d(bdst + off * 128, &mB->box[which], fb, kb * KB, ti.row0 + off, pol_x);
          });
          issued_parity[stage] = static_cast<int>(phase);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
          if (kb == nk - 1) next = atomicAdd(f.tile_counter, 1);   // the next tile, claimed as this one's
        }                                                           // last stage is queued
        if (!ok) break;
      }
      // the end marker: one more stage, no data
      if (!abort_flag && mbar_wait(&empty_bar[stage], phase ^ 1u, &abort_flag, status, wait_ns)) {
        stage_tile[stage] = -1;
        mbar_arrive(&full_bar[stage]);
      }
      if (abort_flag) {   // let every issued copy land before the CTA exits
        for (int i = 0; i < STAGES; ++i)
          if (issued_parity[i] >= 0) mbar_wait_drain(&full_bar[i], static_cast<uint32_t>(issued_parity[i]));
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      for (uint32_t it = 0;; ++it) {
        // the tile whose k-blocks come next: its first stage names it
        if (!mbar_wait(&full_bar[stage], phase, &abort_flag, status, wait_ns)) break;
        const int t = stage_tile[stage];
        if (!mbar_wait(&tmem_empty, (it & 1u) ^ 1u, &abort_flag, status, wait_ns)) break;
        acc_tile = t;
        mbar_arrive(&tile_bar);
        if (t < 0) break;
        int p;
        TileInfo ti;
        locate(t, p, ti);
        const int nk = f.g[p].K / KB;
        const uint32_t idesc = make_idesc(1u, 128u, static_cast<uint32_t>(ti.N));
        const uint32_t d0 = tmem_base;
        tc_fence_after();
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb) {
          if (kb > 0 && !mbar_wait(&full_bar[stage], phase, &abort_flag, status, wait_ns)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA(stage, 0)), a1 = smem_u32(sA(stage, 1));
          const uint32_t b0 = smem_u32(sB(stage));
#pragma unroll
          for (int kk = 0; kk < KB / 16; ++kk) {
            const uint32_t acc = (kb | kk) != 0;
            const uint64_t bd = sw128_desc(b0 + kk * 32);
            umma_bf16(d0, sw128_desc(a0 + kk * 32), bd, idesc, acc);
            umma_bf16(d0 + sub_cols, sw128_desc(a1 + kk * 32), bd, idesc, acc);
          }
          umma_commit(&empty_bar[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(&tmem_full);
      }
      // all issued MMAs must finish before TMEM is released
      umma_commit(&drain_bar);
      mbar_wait_drain(&drain_bar, 0);
    }
  } else {
    // epilogue warps 2 .. 13: warp w reads TMEM lanes 32*(w%4)..+31; down
    // tiles: every third 32-token chunk from (w-2)/4; gate/up tiles: the
    // warps with (w-2)/4 < kGuQ, every kGuQ-th chunk
    const int q = warp & 3;
    const int c0 = (warp - 2) / 4;
    constexpr int cstep = EPIW / 4;
    constexpr int kEpiChunks = (8 + cstep - 1) / cstep;
    const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(32 * q) << 16);
    __nv_bfloat16* stg = stage_out[warp - 2];
    for (uint32_t it = 0;; ++it) {
      if (!mbar_wait(&tile_bar, it & 1u, &abort_flag, status, wait_ns)) break;
      const int t = acc_tile;
      if (t < 0) break;
      int p;
      TileInfo ti;
      const int idx = locate(t, p, ti);
      const GemmArgs& g = f.g[p];
      __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(g.out);
      const size_t out_ld = g.out_ld;
      const int nchunk = (ti.N + 31) / 32;
      float wpre[kEpiChunks];
      if (p >= 2) {                                    // down: routing weights fetched ahead
#pragma unroll
        for (int u = 0; u < kEpiChunks; ++u) {
          const int r = (c0 + u * cstep) * 32 + lane;
          const bool valid = c0 + u * cstep < nchunk && r < ti.n_valid;
          wpre[u] = (g.row_w && valid) ? __ldg(g.row_w + ti.row0 + r) : 0.0f;
        }
      }
      if (!mbar_wait(&tmem_full, it & 1u, &abort_flag, status, wait_ns)) break;
      tc_fence_after();
      if (p < 2) {
        const int feat0 = ti.mb * g.feat_stride + 32 * q;
        for (int c = c0 < kGuQ ? c0 : nchunk; c < nchunk; c += kGuQ) {
          float gv[32], uv[32];
          tmem_ld32(lane_addr + c * 32, gv);
          tmem_ld32(lane_addr + sub_cols + c * 32, uv);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) gv[j] = silu(gv[j]) * uv[j];
          store_tile<32>(stg, gv, lane, out, out_ld, ti.row0 + c * 32, ti.n_valid - c * 32, feat0);
        }
      } else {
#pragma unroll 1
        for (int s = 0; s < 2; ++s) {
          const int feat0 = ti.mb * g.feat_stride + s * g.feat_sub1 + 32 * q;
#pragma unroll
          for (int u = 0; u < kEpiChunks; ++u) {
            const int c = c0 + u * cstep;
            if (c >= nchunk) break;                                  // warp-uniform
            float v[32];
            tmem_ld32(lane_addr + s * sub_cols + c * 32, v);
            tmem_ld_wait();
            if (g.row_w) {
#pragma unroll
              for (int j = 0; j < 32; ++j) v[j] *= __shfl_sync(0xffffffffu, wpre[u], j);
            }
            store_tile<32>(stg, v, lane, out, out_ld, ti.row0 + c * 32, ti.n_valid - c * 32, feat0);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tmem_empty);
      if (p < 2 && c0 < kGuQ) {                        // this warp's part of the h tile is stored
        __threadfence();
        __syncwarp();
        if (lane == 0) atomicAdd(f.ready + idx, 1);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, 512);
}

// ========================================================================
// E4M3 kernel (block-scaled, promotion on CUDA cores), tokens per tile <= 32
// ========================================================================
constexpr int kF8Bn = 32;          // max tokens per tile
constexpr int kF8Slots = 8;        // TMEM ring of per-K-block partial sums
constexpr int kF8SlotCols = 2 * kF8Bn;
constexpr int kF8MaxKb = 64;       // K <= 8192

template <int EPI, int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
grouped_gemm_e4m3_kernel(const __grid_constant__ CUtensorMap tmA,
                         const __grid_constant__ CUtensorMap tmB, const GemmArgs a) {
  constexpr int KB = 128;                          // K elements per stage (128 B)
  constexpr uint32_t A_SUB_BYTES = 128 * 128;
  constexpr uint32_t B_BYTES = kF8Bn * 128;
  constexpr uint32_t STAGE_BYTES = 2 * A_SUB_BYTES + B_BYTES;
  extern __shared__ __align__(1024) uint8_t dsmem[];
  __shared__ Sched sched;
  __shared__ uint64_t full_bar[STAGES], empty_bar[STAGES];
  __shared__ uint64_t part_full[kF8Slots], part_empty[kF8Slots];
  __shared__ uint64_t drain_bar, epi_bar;
  __shared__ uint32_t tmem_base_s;
  __shared__ int issued_parity[STAGES];
  __shared__ volatile int abort_flag;
  __shared__ float bscale_s[kF8Bn * kF8MaxKb];
  __shared__ float red_s[4][kF8Bn];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
  auto sA = [&](int st, int sub) { return smem + st * STAGE_BYTES + sub * A_SUB_BYTES; };
  auto sB = [&](int st) { return smem + st * STAGE_BYTES + 2 * A_SUB_BYTES; };

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 1);
      issued_parity[i] = -1;
    }
    for (int i = 0; i < kF8Slots; ++i) {
      mbar_init(&part_full[i], 1);
      mbar_init(&part_empty[i], 128);
    }
    mbar_init(&drain_bar, 1);
    mbar_init(&epi_bar, 128);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_s, 512);
    tmem_relinquish();
  }
  if (warp == 2) build_schedule(sched, a, lane);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_s;
  const int total = sched.tile_start[a.groups];
  const int nk = a.K / KB;

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol_once = policy_evict_first();
      const uint64_t pol_reuse = policy_evict_normal();
      const uint64_t pol_x = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      for (int t = blockIdx.x; t < total && !abort_flag; t += gridDim.x) {
        const TileInfo ti = decode_tile(sched, a, t);
        const int a_row0 = ti.g * a.a_rows_per_group + ti.mb * a.mblk_stride;
        const int a_row1 = a_row0 + a.sub1_off;
        const uint32_t bytes = 2 * A_SUB_BYTES + B_BYTES;
        const uint64_t pol_w = ti.ntb > 1 ? pol_reuse : pol_once;
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u, &abort_flag, a.status, a.wait_ns)) { ok = false; break; }
          mbar_arrive_expect_tx(&full_bar[stage], bytes);
          tma_load_2d(sA(stage, 0), &tmA, &full_bar[stage], kb * KB, a_row0, pol_w);
          tma_load_2d(sA(stage, 1), &tmA, &full_bar[stage], kb * KB, a_row1, pol_w);
          tma_load_2d(sB(stage), &tmB, &full_bar[stage], kb * KB, ti.row0, pol_x);
          issued_parity[stage] = static_cast<int>(phase);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
      }
      if (abort_flag) {
        for (int i = 0; i < STAGES; ++i)
          if (issued_parity[i] >= 0) mbar_wait_drain(&full_bar[i], static_cast<uint32_t>(issued_parity[i]));
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t kbg = 0;   // K blocks issued so far (TMEM ring position)
      for (int t = blockIdx.x; t < total && !abort_flag; t += gridDim.x) {
        const TileInfo ti = decode_tile(sched, a, t);
        const uint32_t idesc = make_idesc(0u, 128u, static_cast<uint32_t>(ti.N));
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb, ++kbg) {
          const uint32_t slot = kbg % kF8Slots;
          const uint32_t slot_phase = (kbg / kF8Slots) & 1u;
          if (!mbar_wait(&part_empty[slot], slot_phase ^ 1u, &abort_flag, a.status, a.wait_ns)) { ok = false; break; }
          if (!mbar_wait(&full_bar[stage], phase, &abort_flag, a.status, a.wait_ns)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d = tmem_base + slot * kF8SlotCols;
          const uint32_t a0 = smem_u32(sA(stage, 0)), a1 = smem_u32(sA(stage, 1));
          const uint32_t b0 = smem_u32(sB(stage));
#pragma unroll
          for (int kk = 0; kk < KB / 32; ++kk) {
            const uint64_t bd = sw128_desc(b0 + kk * 32);
            umma_e4m3(d, sw128_desc(a0 + kk * 32), bd, idesc, kk != 0);
            umma_e4m3(d + kF8Bn, sw128_desc(a1 + kk * 32), bd, idesc, kk != 0);
          }
          umma_commit(&empty_bar[stage]);
          umma_commit(&part_full[slot]);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
      }
      umma_commit(&drain_bar);
      mbar_wait_drain(&drain_bar, 0);
    }
  } else {
    const int q = warp & 3;
    const int et = threadIdx.x - 64;            // 0..127
    const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(32 * q) << 16);
    const int nkb_a = a.K / 128;
    const int a_blk_rows = a.a_rows_per_group / 128;
    uint32_t kbg = 0, epi_phase = 0;
    bool ok = true;
    // Bounded sync of the 128 epilogue threads (an abort ends it, never hangs).
    auto epi_sync = [&]() -> bool {
      mbar_arrive(&epi_bar);
      const bool r = mbar_wait(&epi_bar, epi_phase, &abort_flag, a.status, a.wait_ns);
      epi_phase ^= 1u;
      return r;
    };
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
      const TileInfo ti = decode_tile(sched, a, t);
      // activation scales of this tile's rows -> smem
      if (!epi_sync()) break;
      for (int i = et; i < kF8Bn * nk; i += 128) {
        const int r = i / nk, kb = i - r * nk;
        bscale_s[r * kF8MaxKb + kb] = (r < ti.n_valid) ? a.b_scale[static_cast<size_t>(ti.row0 + r) * nk + kb] : 0.0f;
      }
      if (!epi_sync()) break;
      const int a_row0 = ti.g * a.a_rows_per_group + ti.mb * a.mblk_stride;
      const int a_row1 = a_row0 + a.sub1_off;
      const float* as_g = a.a_scale + static_cast<size_t>(ti.g) * a_blk_rows * nkb_a;
      const float* as0 = as_g + static_cast<size_t>((a_row0 - ti.g * a.a_rows_per_group) / 128) * nkb_a;
      const float* as1 = as_g + static_cast<size_t>((a_row1 - ti.g * a.a_rows_per_group) / 128) * nkb_a;
      float acc0[kF8Bn], acc1[kF8Bn];
#pragma unroll
      for (int j = 0; j < kF8Bn; ++j) { acc0[j] = 0.f; acc1[j] = 0.f; }
      for (int kb = 0; kb < nk; ++kb, ++kbg) {
        const uint32_t slot = kbg % kF8Slots;
        const uint32_t slot_phase = (kbg / kF8Slots) & 1u;
        if (!mbar_wait(&part_full[slot], slot_phase, &abort_flag, a.status, a.wait_ns)) { ok = false; break; }
        tc_fence_after();
        float v0[32], v1[32];
        tmem_ld32(lane_addr + slot * kF8SlotCols, v0);
        tmem_ld32(lane_addr + slot * kF8SlotCols + kF8Bn, v1);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&part_empty[slot]);
        const float s0 = __ldg(as0 + kb), s1 = __ldg(as1 + kb);
#pragma unroll
        for (int j = 0; j < kF8Bn; ++j) {
          const float sb = bscale_s[j * kF8MaxKb + kb];
          acc0[j] = fmaf(v0[j], s0 * sb, acc0[j]);
          acc1[j] = fmaf(v1[j], s1 * sb, acc1[j]);
        }
      }
      if (!ok) break;
      if (EPI == EPI_SWIGLU) {
        // h for feature mb*128 + (this thread's TMEM lane), tokens j;
        // 1x128 quantisation along I (the 128 lanes of the tile)
        const int feat = ti.mb * a.feat_stride + 32 * q + lane;
        float h[kF8Bn];
#pragma unroll
        for (int j = 0; j < kF8Bn; ++j) {
          h[j] = silu(acc0[j]) * acc1[j];
          float m = fabsf(h[j]);
#pragma unroll
          for (int d = 16; d > 0; d >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, d));
          if (lane == 0) red_s[q][j] = m;
        }
        if (!epi_sync()) break;
        uint8_t* outq = reinterpret_cast<uint8_t*>(a.out);
        const int nsc = a.out_ld / 128;
#pragma unroll
        for (int j = 0; j < kF8Bn; ++j) {
          if (j < ti.n_valid) {
            const float amax = fmaxf(fmaxf(red_s[0][j], red_s[1][j]), fmaxf(red_s[2][j], red_s[3][j]));
            const float sc = amax == 0.0f ? 1.0f : amax / 448.0f;
            outq[static_cast<size_t>(ti.row0 + j) * a.out_ld + feat] = to_e4m3(h[j] / sc);
            if (et == j) a.out_scale[static_cast<size_t>(ti.row0 + j) * nsc + ti.mb] = sc;
          }
        }
      } else {
        __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(a.out);
        const int f0 = ti.mb * a.feat_stride + 32 * q + lane;
        const int f1 = f0 + a.feat_sub1;
#pragma unroll
        for (int j = 0; j < kF8Bn; ++j) {
          if (j < ti.n_valid) {
            const float w = a.row_w ? __ldg(a.row_w + ti.row0 + j) : 1.0f;
            const size_t r = static_cast<size_t>(ti.row0 + j) * a.out_ld;
            out[r + f0] = __float2bfloat16_rn(acc0[j] * w);
            out[r + f1] = __float2bfloat16_rn(acc1[j] * w);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, 512);
}

// ------------------------------------------------------------------------
// host-side launch helpers (called from api.cu)
// ------------------------------------------------------------------------
size_t gemm_bf16_smem_bytes(int bn_max) {
  return static_cast<size_t>(kBf16Stages) * (2 * 128 * 128 + static_cast<size_t>(bn_max) * 128) + 1024;
}
size_t gemm_e4m3_smem_bytes() {
  return static_cast<size_t>(kE4m3Stages) * (2 * 128 * 128 + kF8Bn * 128) + 1024;
}

using Bf16Kernel = void (*)(CUtensorMap, TokenMaps, GemmArgs, CUtensorMap, TokenMaps, GemmArgs);

// The bf16 kernel forms: (one problem | two) x (4 | 12 epilogue warps).
template <int EPI>
Bf16Kernel bf16_kernel(bool two, int epi_warps) {
  if (epi_warps == 12)
    return two ? grouped_gemm_bf16_kernel<EPI, kBf16Stages, false, true, 12>
               : grouped_gemm_bf16_kernel<EPI, kBf16Stages, false, false, 12>;
  return two ? grouped_gemm_bf16_kernel<EPI, kBf16Stages, false, true, 4>
             : grouped_gemm_bf16_kernel<EPI, kBf16Stages, false, false, 4>;
}

cudaError_t launch_grouped_gemm(bool e4m3, int epi, const CUtensorMap& tmA, const TokenMaps& tmB,
                                const GemmArgs& a, int grid, cudaStream_t stream, const SecondProblem* two) {
  if (!e4m3) {
    const bool gather = a.gather_rows != nullptr;
    const int epiw = gather ? 4 : (a.epi_warps == 12 ? 12 : 4);
    const int threads = 64 + 32 * epiw + (gather ? kGatherThreads : 0);
    const size_t smem = gemm_bf16_smem_bytes(a.bn_max);
    const bool pair2 = two != nullptr && !gather;
    Bf16Kernel kern;
    if (gather)
      kern = epi == EPI_SWIGLU ? grouped_gemm_bf16_kernel<EPI_SWIGLU, kBf16Stages, true, false>
                               : grouped_gemm_bf16_kernel<EPI_WEIGHTED, kBf16Stages, true, false>;
    else if (epi == EPI_SCATTER)
      kern = bf16_kernel<EPI_SCATTER>(pair2, epiw);
    else
      kern = epi == EPI_SWIGLU ? bf16_kernel<EPI_SWIGLU>(pair2, epiw) : bf16_kernel<EPI_WEIGHTED>(pair2, epiw);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    if (pair2)
      kern<<<grid, threads, smem, stream>>>(tmA, tmB, a, two->tmA, two->tmB, two->a);
    else
      kern<<<grid, threads, smem, stream>>>(tmA, tmB, a, tmA, tmB, a);
  } else {
    const size_t smem = gemm_e4m3_smem_bytes();
    auto kern = epi == EPI_SWIGLU ? grouped_gemm_e4m3_kernel<EPI_SWIGLU, kE4m3Stages>
                                  : grouped_gemm_e4m3_kernel<EPI_WEIGHTED, kE4m3Stages>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    kern<<<grid, kThreads, smem, stream>>>(tmA, tmB.box[0], a);
  }
  return cudaGetLastError();
}

cudaError_t launch_ffn_bf16(const FfnArgs& f, int grid, cudaStream_t stream) {
  const size_t smem = gemm_bf16_smem_bytes(f.g[1].bn_max);
  cudaError_t e = cudaFuncSetAttribute(grouped_ffn_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  grouped_ffn_bf16_kernel<<<grid, 64 + 32 * kFfnEpiWarps, smem, stream>>>(f);
  return cudaGetLastError();
}

}  // namespace moe
