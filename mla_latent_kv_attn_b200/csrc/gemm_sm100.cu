// gemm_sm100.cu - bf16 GEMM on the 5th-generation tensor cores for the projections of the
// path (joint query/KV down-projection, absorbed query heads, value up-projection, W_O).
//
//   C[z](m, n) = sum_k A[z](m, k) * B[z](n, k)     bf16 operands, fp32 accumulation in TMEM
//
// Persistent: a grid of at most one CTA per SM walks the 128 x BN output tiles (tile index
// n-fastest, so CTAs working at the same time share the A rows through L2), each CTA taking
// every gridDim.x-th tile.  Roles (320 threads):
//   warp 0     TMA producer: 128x64 (A) and BNx64 (B) K-slices into a ring of 128B-swizzled
//              buffers as deep as shared memory allows (4 to 8 stages); the ring runs on across
//              tile boundaries.
//   warp 1     allocates TMEM; one thread issues tcgen05.mma (M=128, N=BN, K=16) into one of two
//              TMEM accumulators (tiles alternate), committing each stage back to the producer
//              and each finished accumulator to the epilogue.
//   warps 2-9  epilogue, two groups of four warps (each group one TMEM lane = one output row per
//              thread, group g taking the 32-column chunks 2k + g): drain an accumulator,
//              optionally rotate the positional-query columns (the last d_rope columns of every
//              head block: 3D-RoPE), write bf16 into a 64B-swizzled 128x32 staging buffer (two
//              per group, alternating) that one thread of the group stores with a TMA
//              bulk-tensor store (whole lines, out-of-range rows and columns clipped), and hand
//              the accumulator back; this overlaps the MMAs of the CTA's next tile.  Outputs whose
//              strides TMA cannot take are stored row by row.  (With one group, one warp per
//              sub-partition, the drain took longer than the next tile's main loop.)
// Before the first K-slice of a tile the producer asks L2 for its share of the tile's A panel
// (when the panel is one contiguous range) with one bulk prefetch, so the panel streams from HBM
// in long runs instead of one 128-byte piece per row and K-slice.
// Optionally the columns n >= n_split go to a second output C2 (column n - n_split): one GEMM
// over [W_1; W_2] then writes x W_1^T and x W_2^T to their own arrays.  Optionally every output
// row is also stored into a ring of frames (the fused down-projection and cache append), and
// optionally the epilogue writes the rotated positional keys the chunk's attention reads (the
// chunk's own from the k_R columns of each row, the ring's from the cache while the first
// tile's MMAs run), so that attention needs no separate rotation pass.
// Launched with programmatic serialisation (launch_pdl): barrier set-up and the TMEM allocation
// may overlap the previous kernel's tail.
#include "kernels.h"
#include "sm100.cuh"

namespace mla {

namespace {

using namespace sm100;

constexpr int kBM = 128;
constexpr int kBK = 64;          // one 128-byte swizzle atom of bf16 per row
constexpr int kThreads = 320;    // 10 warps
constexpr int kEpiThreads = 256; // two groups of four warps, each group all 128 TMEM lanes
constexpr int kEpiGroupThreads = 128;

constexpr int kMaxStages = 8;
constexpr int kEpiCols = 32;                       // columns per staged store
constexpr int kStageOut = kBM * kEpiCols * 2;      // 8 KB: one 128 x 32 bf16 staging buffer
constexpr int kStagingBufs = 4;                    // two per epilogue group
constexpr int kSmemBudget = 220 * 1024 - kStagingBufs * kStageOut;   // for the operand ring

template <int BN>
struct GemmCfg {
  static constexpr int kATile = kBM * kBK * 2;
  static constexpr int kBTile = BN * kBK * 2;
  static constexpr int kStage = kATile + kBTile;
  // As many stages as fit: the loads in flight per SM must cover the L2/HBM latency.
  static constexpr int kStages = kSmemBudget / kStage < kMaxStages ? kSmemBudget / kStage : kMaxStages;
  static constexpr int kOut = kStages * kStage;          // staging buffers after the ring
  static constexpr int kSmem = kOut + kStagingBufs * kStageOut + 1024;  // + slack to align
  // two accumulators, each starting on a power-of-two column
  static constexpr int kAccStride = BN <= 32 ? 32 : BN <= 64 ? 64 : BN <= 128 ? 128 : 256;
  static constexpr int kTmemCols = 2 * kAccStride;
  static_assert(BN <= 256 && BN % 16 == 0, "tcgen05 M=128 needs N a multiple of 16 up to 256");
};

struct GemmParams {
  int M, N, K, batch;
  int n_tiles_m, n_tiles_n;
  int a_swapped, b_swapped;  // tensor map dims are (K, batch, rows) instead of (K, rows, batch)
  void* C;
  int64_t c_sm, c_batch;
  void* C2;                  // columns >= n_split (0 = no split)
  int64_t c2_sm, c2_batch;
  int n_split;
  int tma_store;             // 1: stores through tmC / tmC2 (see launch_gemm)
  int c_swapped, c2_swapped; // output maps are (N, batch, rows) instead of (N, rows, batch)
  int prefetch_a;            // 1: the A panel of a tile is one contiguous range
  const void* A;
  int64_t a_sm;
  int epilogue;
  int rope_D, rope_dr, rope_n_q, rope_first_frame;
  RopeGeom rope;
  bf16* ring;                // ring append (see TcGemmArgs), or null
  int32_t* slot_frame;
  int ring_W, ring_tpf, ring_n_q, ring_first, ring_B;
  bf16* rk;                  // rotated positional keys (see TcGemmArgs), or null
  const bf16* rk_cache;
  const int32_t* rk_slot_frame;
  int32_t* rk_dev_status;
  int rk_col, rk_dr, rk_D, rk_dc, rk_n_q, rk_B, rk_W, rk_nc, rk_nc_pad, rk_rows, rk_first, rk_ring;
};

// Row r of sample b of the rotated-key workspace (ring slot, padding or tail row).
__device__ __forceinline__ void gemm_key_row(const GemmParams& p, int b, int r) {
  switch (p.rk_dr) {
#define MLA_GEMM_KEY_ROW(DR)                                                                     \
  case DR:                                                                                       \
    rope_key_row<bf16, DR / 8>(p.rk_cache, nullptr, p.rk_slot_frame, p.rk, b, r, p.rk_W, p.rk_D, \
                               p.rk_dc, p.rk_n_q, p.rk_nc, p.rk_nc_pad, p.rk_rows, p.rk_first,   \
                               p.rope, p.rk_dev_status, 1);                                      \
    break;
    MLA_GEMM_KEY_ROW(16)
    MLA_GEMM_KEY_ROW(32)
    MLA_GEMM_KEY_ROW(64)
#undef MLA_GEMM_KEY_ROW
    default: break;
  }
}

// Sine and cosine of the rotary pairs of the rotated-key chunk at output column n (rk_col <= n <
// rk_col + rk_dr, a multiple of 32) for row m = chunk token j of sample m / rk_n_q, at frame
// rk_first + j / tpf.  They depend on the row's position only, so the epilogue computes them
// before the tile's accumulator is ready.
__device__ __forceinline__ void gemm_key_sincos(const GemmParams& p, int m, int n, float* sn,
                                                float* cs) {
  const int j = m % p.rk_n_q;
  const int i = j % p.rope.tpf;
  const int t = p.rk_first + j / p.rope.tpf, h = i / p.rope.frame_w, w = i % p.rope.frame_w;
  const int c0 = n - p.rk_col;
  const int npairs = min(16, (p.rk_dr - c0) / 2);    // 8 or 16
#pragma unroll
  for (int pr = 0; pr < 16; ++pr) {
    sn[pr] = 0.f;
    cs[pr] = 1.f;
    if (pr < npairs) rope_sincos(rope_angle(p.rope, c0 / 2 + pr, t, h, w), &sn[pr], &cs[pr]);
  }
}

// The chunk token's rotated positional key from the 32 accumulator columns v of the epilogue
// chunk at output column n, with its pairs' sine and cosine from gemm_key_sincos: each value is
// taken as chunk_lat stores it (rounded to bf16), rotated in fp32 and rounded once, as
// rope_key_row does.
__device__ __forceinline__ void gemm_chunk_key(const GemmParams& p, int m, int n, const float* v,
                                               const float* sn, const float* cs) {
  const int bs = m / p.rk_n_q, j = m % p.rk_n_q;
  const int c0 = n - p.rk_col;                       // a multiple of 32
  const int npairs = min(16, (p.rk_dr - c0) / 2);    // 8 or 16
  uint32_t packed[16];
#pragma unroll
  for (int pr = 0; pr < 16; ++pr) {
    float x0 = __bfloat162float(__float2bfloat16_rn(v[2 * pr]));
    float x1 = __bfloat162float(__float2bfloat16_rn(v[2 * pr + 1]));
    rope_apply(x0, x1, sn[pr], cs[pr]);
    packed[pr] = pack_bf16x2(x0, x1);
  }
  uint4* d4 = reinterpret_cast<uint4*>(
      p.rk + (static_cast<int64_t>(bs) * p.rk_rows + p.rk_nc_pad + j) * p.rk_dr + c0);
#pragma unroll
  for (int q = 0; q < 4; ++q)
    if (4 * q < npairs)
      d4[q] = make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
}

__device__ __forceinline__ void store_row32(bf16* dst, const float* v, int valid, bool vec_ok) {
  if (vec_ok && valid >= 32) {
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) w[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
    uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int i = 0; i < 4; ++i) d4[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (i < valid) dst[i] = __float2bfloat16_rn(v[i]);
  }
}

struct TileCoord {
  int z, m0, n0;
};

__device__ __forceinline__ TileCoord tile_coord(const GemmParams& p, int t) {
  TileCoord c;
  const int per_z = p.n_tiles_m * p.n_tiles_n;
  c.z = t / per_z;
  const int r = t - c.z * per_z;
  c.m0 = (r / p.n_tiles_n) * kBM;
  c.n0 = (r % p.n_tiles_n);
  return c;
}

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmC2,
                   GemmParams p) {
  using Cfg = GemmCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  constexpr int kStages = Cfg::kStages;
  __shared__ __align__(8) uint64_t full_bar[kStages];
  __shared__ __align__(8) uint64_t empty_bar[kStages];
  __shared__ __align__(8) uint64_t acc_full[2];
  __shared__ __align__(8) uint64_t acc_empty[2];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int nkb = ceil_div(p.K, kBK);
  const int n_tiles = p.n_tiles_m * p.n_tiles_n * p.batch;
  volatile int* abort_flag = &abort_sh;

  if (threadIdx.x == 0) {
    abort_sh = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&acc_full[a]), 1);
      mbar_init(smem_u32(&acc_empty[a]), kEpiThreads);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_base_sh), Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  grid_dep_wait();     // the previous kernel on the stream has completed (programmatic launch)
  grid_dep_launch();

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
        const TileCoord tc = tile_coord(p, t);
        const int n0 = tc.n0 * BN;
        if (p.prefetch_a) {
          // share tc.n0 of n_tiles_n of the rows m0 .. m0+127 (all of K, contiguous)
          const int rows = min(kBM, p.M - tc.m0);
          const int r0 = rows * tc.n0 / p.n_tiles_n, r1 = rows * (tc.n0 + 1) / p.n_tiles_n;
          const uint32_t row_bytes = static_cast<uint32_t>(p.a_sm) * 2u;
          if (r1 > r0)
            prefetch_l2_bulk(static_cast<const uint8_t*>(p.A) +
                                 static_cast<int64_t>(tc.m0 + r0) * row_bytes,
                             static_cast<uint32_t>(r1 - r0) * row_bytes);
        }
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1;
          ok = mbar_wait_or_abort(smem_u32(&empty_bar[s]), ph ^ 1, abort_flag, nullptr);
          if (!ok) break;
          const uint32_t a_dst = base + s * Cfg::kStage;
          const uint32_t b_dst = a_dst + Cfg::kATile;
          const uint32_t fb = smem_u32(&full_bar[s]);
          mbar_arrive_expect_tx(fb, Cfg::kStage);
          if (p.a_swapped) tma_load_3d(a_dst, &tmA, fb, kb * kBK, tc.z, tc.m0);
          else tma_load_3d(a_dst, &tmA, fb, kb * kBK, tc.m0, tc.z);
          if (p.b_swapped) tma_load_3d(b_dst, &tmB, fb, kb * kBK, tc.z, n0);
          else tma_load_3d(b_dst, &tmB, fb, kb * kBK, n0, tc.z);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kBM, BN, 0, 0);
      int it = 0, lt = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++lt) {
        const int acc = lt & 1;
        // the epilogue has drained this accumulator (its previous tile); first use passes
        ok = mbar_wait_or_abort(smem_u32(&acc_empty[acc]), ((lt >> 1) & 1) ^ 1, abort_flag, nullptr);
        if (!ok) break;
        tc_fence_after();
        const uint32_t d = tmem + acc * Cfg::kAccStride;
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1;
          ok = mbar_wait_or_abort(smem_u32(&full_bar[s]), ph, abort_flag, nullptr);
          if (!ok) break;
          tc_fence_after();
          const uint32_t a_addr = base + s * Cfg::kStage;
          const uint32_t b_addr = a_addr + Cfg::kATile;
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            const uint64_t ad = smem_desc(a_addr + 32 * k, 16, 1024, kSwizzle128B);
            const uint64_t bd = smem_desc(b_addr + 32 * k, 16, 1024, kSwizzle128B);
            mma_ss(d, ad, bd, idesc, (kb | k) != 0 ? 1u : 0u);
          }
          mma_commit(smem_u32(&empty_bar[s]));
        }
        if (ok) mma_commit(smem_u32(&acc_full[acc]));
      }
    }
  } else {
    // epilogue warps 2..9: group 0 = warps 2..5, group 1 = warps 6..9, each covering TMEM lane
    // quadrants 2, 3, 0, 1; group g drains the 32-column chunks 2k + g of every tile (two
    // groups, because one warp per sub-partition leaves the TMEM loads' latency exposed)
    const int quad = warp & 3;
    const int grp = (warp - 2) >> 2;
    const int row = quad * 32 + lane;
    const bool leader = threadIdx.x == 64 + kEpiGroupThreads * grp;   // issues the TMA stores
    const uint32_t out_base = base + Cfg::kOut + grp * 2 * kStageOut;
    const bool vec_ok = ((reinterpret_cast<uintptr_t>(p.C) & 15u) == 0) && (p.c_sm % 8 == 0) &&
                        (p.c_batch % 8 == 0) &&
                        (p.n_split == 0 || (((reinterpret_cast<uintptr_t>(p.C2) & 15u) == 0) &&
                                            (p.c2_sm % 8 == 0) && (p.c2_batch % 8 == 0)));
    if (p.ring != nullptr && blockIdx.x == 0 && threadIdx.x == 64) {
      // the appended frames' slots: frame first + j of every sample lands in slot (first+j) mod W
      const int frames = p.ring_n_q / p.ring_tpf;
      for (int e = 0; e < p.ring_B * frames; ++e) {
        const int f = p.ring_first + e % frames;
        p.slot_frame[(e / frames) * p.ring_W + f % p.ring_W] = f;
      }
    }
    const bool ring_vec = p.ring != nullptr && ((reinterpret_cast<uintptr_t>(p.ring) & 15u) == 0) &&
                          (p.N % 8 == 0);
    if (p.rk != nullptr) {
      // the rotated-key rows that do not come from this GEMM's output: the ring part (with
      // rk_ring) and the zero rows after the chunk, spread over every epilogue thread of the grid
      // while the first tile's MMAs run
      const int ring_rows = p.rk_ring ? p.rk_nc_pad : 0;
      const int tail0 = p.rk_nc_pad + p.rk_n_q;
      const int per = ring_rows + (p.rk_rows - tail0);
      const int total = p.rk_B * per;                // < 2^31 (host check)
      for (int e = blockIdx.x * kEpiThreads + (threadIdx.x - 64); e < total;
           e += gridDim.x * kEpiThreads) {
        const int b = e / per, i = e % per;
        gemm_key_row(p, b, i < ring_rows ? i : tail0 + (i - ring_rows));
      }
    }
    int lt = 0, chunk = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++lt) {
      const int acc = lt & 1;
      // the rotated-key chunk this group drains in this tile, if any (output column rk_n), with
      // its rotary sines and cosines for this thread's row, while the tile's MMAs run
      int rk_n = -1;
      float rk_sin[16], rk_cos[16];
      if (p.rk != nullptr) {
        const TileCoord tk = tile_coord(p, t);
        const int kn0 = tk.n0 * BN;
        for (int c = p.rk_col; c < p.rk_col + p.rk_dr; c += kEpiCols)
          if (c >= kn0 && c < kn0 + BN && (((c - kn0) / kEpiCols) & 1) == grp) rk_n = c;
        if (rk_n >= 0 && tk.m0 + row < p.M) gemm_key_sincos(p, tk.m0 + row, rk_n, rk_sin, rk_cos);
      }
      const bool ok = __all_sync(0xffffffffu, mbar_wait_or_abort(smem_u32(&acc_full[acc]),
                                                                  (lt >> 1) & 1, abort_flag, nullptr));
      if (!ok) break;
      tc_fence_after();
      const TileCoord tc = tile_coord(p, t);
      const int n0 = tc.n0 * BN;
      const int m = tc.m0 + row;
      int t_pos = 0, hh = 0, ww = 0;
      if (p.epilogue == kEpiRopeQ) {
        const int nl = m % p.rope_n_q;
        const int i = nl % p.rope.tpf;
        t_pos = p.rope_first_frame + nl / p.rope.tpf;
        hh = i / p.rope.frame_w;
        ww = i % p.rope.frame_w;
      }
      const uint32_t tacc = tmem + (static_cast<uint32_t>(quad * 32) << 16) + acc * Cfg::kAccStride;
#pragma unroll 1
      for (int c0 = kEpiCols * grp; c0 < BN; c0 += 2 * kEpiCols, ++chunk) {
        const int n = n0 + c0;
        if (n >= p.N) break;                   // uniform over the CTA
        uint32_t r[32];
        tmem_ld32_wait(tacc + c0, r);
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
        if (p.epilogue == kEpiRopeQ) {
          // columns rope0 .. D-1 of every D-wide head block are the positional query; a 32-column
          // chunk may start anywhere in a head block (D is a multiple of 16, not of 32)
          const int cb0 = n % p.rope_D;
          const int rope0 = p.rope_D - p.rope_dr;
          if (cb0 + 32 > rope0) {
#pragma unroll
            for (int pr = 0; pr < 16; ++pr) {
              const int cb = cb0 + 2 * pr;
              if (cb >= rope0 && cb < p.rope_D)
                rope_rotate(v[2 * pr], v[2 * pr + 1],
                            rope_angle(p.rope, (cb - rope0) >> 1, t_pos, hh, ww));
            }
          }
        }
        const bool second = p.n_split > 0 && n >= p.n_split;
        if (n == rk_n && m < p.M) gemm_chunk_key(p, m, n, v, rk_sin, rk_cos);
        if (p.ring != nullptr && m < p.M) {
          // the same row into its ring slot (whole frames wrap; row width N)
          const int bs = m / p.ring_n_q, r = m % p.ring_n_q;
          const int slot = (p.ring_first + r / p.ring_tpf) % p.ring_W;
          bf16* rrow = p.ring + (static_cast<int64_t>(bs) * p.ring_W * p.ring_tpf +
                                 static_cast<int64_t>(slot) * p.ring_tpf + r % p.ring_tpf) * p.N;
          store_row32(rrow + n, v, p.N - n, ring_vec);
        }
        if (p.tma_store) {
          const uint32_t buf = out_base + (chunk & 1) * kStageOut;
          // the store that last read this buffer (two chunks ago) has finished reading it
          if (leader) bulk_wait_group_read<1>();
          named_bar_sync(1 + grp, kEpiGroupThreads);
          // row `row` is 64 B: four 16-byte pieces, piece j at j ^ ((row / 2) mod 4) (64B swizzle)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint4 w4 = make_uint4(pack_bf16x2(v[8 * j + 0], v[8 * j + 1]),
                                        pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                                        pack_bf16x2(v[8 * j + 4], v[8 * j + 5]),
                                        pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
            const uint32_t dst = buf + row * 64 + ((j ^ ((row >> 1) & 3)) << 4);
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(w4.x),
                         "r"(w4.y), "r"(w4.z), "r"(w4.w)
                         : "memory");
          }
          fence_proxy_async_smem();
          named_bar_sync(1 + grp, kEpiGroupThreads);
          if (leader) {
            const CUtensorMap* map = second ? &tmC2 : &tmC;
            const int col = second ? n - p.n_split : n;
            if (second ? p.c2_swapped : p.c_swapped) tma_store_3d(map, buf, col, tc.z, tc.m0);
            else tma_store_3d(map, buf, col, tc.m0, tc.z);
            bulk_commit_group();
          }
        } else if (m < p.M) {
          if (second) {
            bf16* crow = static_cast<bf16*>(p.C2) + static_cast<int64_t>(tc.z) * p.c2_batch +
                         static_cast<int64_t>(m) * p.c2_sm;
            store_row32(crow + (n - p.n_split), v, p.N - n, vec_ok);
          } else {
            bf16* crow = static_cast<bf16*>(p.C) + static_cast<int64_t>(tc.z) * p.c_batch +
                         static_cast<int64_t>(m) * p.c_sm;
            store_row32(crow + n, v, (p.n_split > 0 ? p.n_split : p.N) - n, vec_ok);
          }
        }
      }
      // accumulator drained: the MMA thread may start the CTA's next-but-one tile in it
      tc_fence_before();
      mbar_arrive(smem_u32(&acc_empty[acc]));
    }
    if (leader) bulk_wait_group_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

// Tensor map over one bf16 matrix [batch][rows, cols] (cols contiguous), box (box_cols,
// box_rows, 1).  TMA wants increasing strides, so when the batch stride is below the row stride
// the map is built over (cols, batch, rows) and *swapped is set.
mla_status matrix_map(CUtensorMap* map, const void* base, int cols, int rows, int batch,
                      int64_t row_stride, int64_t batch_stride, uint32_t box_cols,
                      uint32_t box_rows, int swizzle, int* swapped) {
  const int64_t bs = batch > 1 ? batch_stride : row_stride * rows;
  *swapped = (batch > 1 && bs < row_stride) ? 1 : 0;
  if (*swapped) {
    const uint64_t dims[3] = {static_cast<uint64_t>(cols), static_cast<uint64_t>(batch),
                              static_cast<uint64_t>(rows)};
    const uint64_t strides[2] = {static_cast<uint64_t>(bs) * 2, static_cast<uint64_t>(row_stride) * 2};
    const uint32_t box[3] = {box_cols, 1, box_rows};
    return make_tmap_bf16(map, base, 3, dims, strides, box, swizzle);
  }
  const uint64_t dims[3] = {static_cast<uint64_t>(cols), static_cast<uint64_t>(rows),
                            static_cast<uint64_t>(batch)};
  const uint64_t strides[2] = {static_cast<uint64_t>(row_stride) * 2, static_cast<uint64_t>(bs) * 2};
  const uint32_t box[3] = {box_cols, box_rows, 1};
  return make_tmap_bf16(map, base, 3, dims, strides, box, swizzle);
}

mla_status operand_map(CUtensorMap* map, const void* base, int K, int rows, int batch,
                       int64_t row_stride, int64_t batch_stride, uint32_t box_rows, int* swapped) {
  return matrix_map(map, base, K, rows, batch, row_stride, batch_stride, kBK, box_rows, 128, swapped);
}

// An output can take TMA stores when its base is 16-byte aligned and its strides are whole
// multiples of 16 bytes.
bool tma_storable(const void* c, int64_t c_sm, int64_t c_batch, int batch) {
  return (reinterpret_cast<uintptr_t>(c) & 15u) == 0 && c_sm % 8 == 0 &&
         (batch == 1 || c_batch % 8 == 0);
}

int num_sms() {
  static int n = [] {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) {
      cudaGetLastError();
      return 148;
    }
    return v;
  }();
  return n;
}

template <int BN>
mla_status launch_gemm(const TcGemmArgs& g, cudaStream_t s) {
  using Cfg = GemmCfg<BN>;
  CUtensorMap ta, tb;
  int a_sw = 0, b_sw = 0;
  mla_status st = operand_map(&ta, g.A, g.K, g.M, g.batch, g.a_sm, g.a_batch, kBM, &a_sw);
  if (st != MLA_OK) return st;
  st = operand_map(&tb, g.B, g.K, g.N, g.batch, g.b_sn, g.b_batch, BN, &b_sw);
  if (st != MLA_OK) return st;
  GemmParams p;
  p.M = g.M; p.N = g.N; p.K = g.K; p.batch = g.batch;
  p.n_tiles_m = ceil_div(g.M, kBM); p.n_tiles_n = ceil_div(g.N, BN);
  p.a_swapped = a_sw; p.b_swapped = b_sw;
  p.C = g.C; p.c_sm = g.c_sm; p.c_batch = g.c_batch;
  p.C2 = g.C2; p.c2_sm = g.c2_sm; p.c2_batch = g.c2_batch; p.n_split = g.n_split;
  p.epilogue = g.epilogue; p.rope_D = g.rope_D; p.rope_dr = g.rope_dr; p.rope_n_q = g.rope_n_q;
  p.rope_first_frame = g.rope_first_frame; p.rope = g.rope;
  p.A = g.A; p.a_sm = g.a_sm;
  p.prefetch_a = (g.batch == 1 && g.a_sm == g.K) ? 1 : 0;
  p.ring = static_cast<bf16*>(g.ring); p.slot_frame = g.slot_frame;
  p.ring_W = g.ring_W; p.ring_tpf = g.ring_tpf; p.ring_n_q = g.ring_n_q;
  p.ring_first = g.ring_first; p.ring_B = g.ring_B;
  p.rk = static_cast<bf16*>(g.rk); p.rk_cache = static_cast<const bf16*>(g.rk_cache);
  p.rk_slot_frame = g.rk_slot_frame; p.rk_dev_status = g.rk_dev_status;
  p.rk_col = g.rk_col; p.rk_dr = g.rk_dr; p.rk_D = g.rk_D; p.rk_dc = g.rk_dc;
  p.rk_n_q = g.rk_n_q; p.rk_B = g.rk_B; p.rk_W = g.rk_W; p.rk_nc = g.rk_nc;
  p.rk_nc_pad = g.rk_nc_pad; p.rk_rows = g.rk_rows; p.rk_first = g.rk_first;
  p.rk_ring = g.rk_ring;
  // output maps: 32 x 128 boxes, 64B swizzle (the staging layout)
  CUtensorMap tc, tc2;
  p.tma_store = tma_storable(g.C, g.c_sm, g.c_batch, g.batch) &&
                (g.n_split == 0 || tma_storable(g.C2, g.c2_sm, g.c2_batch, g.batch));
  p.c_swapped = p.c2_swapped = 0;
  if (p.tma_store) {
    const int n1 = g.n_split > 0 ? g.n_split : g.N;
    st = matrix_map(&tc, g.C, n1, g.M, g.batch, g.c_sm, g.c_batch, kEpiCols, kBM, 64, &p.c_swapped);
    if (st != MLA_OK) return st;
    if (g.n_split > 0) {
      st = matrix_map(&tc2, g.C2, g.N - g.n_split, g.M, g.batch, g.c2_sm, g.c2_batch, kEpiCols,
                      kBM, 64, &p.c2_swapped);
      if (st != MLA_OK) return st;
    } else {
      tc2 = tc;   // never used
    }
  } else {
    tc = ta;      // never used
    tc2 = ta;
  }
  MLA_CUDA_TRY(cudaFuncSetAttribute(gemm_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    Cfg::kSmem));
  const long long tiles = static_cast<long long>(p.n_tiles_m) * p.n_tiles_n * g.batch;
  const int grid = static_cast<int>(std::min<long long>(tiles, num_sms()));
  MLA_CUDA_TRY(launch_pdl(gemm_tc_kernel<BN>, dim3(grid), dim3(kThreads), Cfg::kSmem, s, ta, tb,
                          tc, tc2, p));
  return MLA_OK;
}

}  // namespace

bool tc_gemm_supported(int M, int N, int K, int64_t a_sm, int64_t b_sn) {
  return M > 0 && N > 0 && K > 0 && K % 8 == 0 && a_sm % 8 == 0 && b_sn % 8 == 0;
}

mla_status gemm_tc(const TcGemmArgs& g, cudaStream_t s) {
  if (g.M == 0 || g.N == 0) return MLA_OK;
  if (g.n_split != 0 && (g.n_split % 32 != 0 || g.n_split >= g.N || g.C2 == nullptr))
    MLA_FAIL(MLA_ERR_INVALID_ARG, "GEMM column split must be a multiple of 32 inside N");
  if (g.ring != nullptr &&
      (g.batch != 1 || g.n_split != 0 || g.slot_frame == nullptr || g.ring_W <= 0 ||
       g.ring_tpf <= 0 || g.ring_n_q % g.ring_tpf != 0 ||
       static_cast<int64_t>(g.ring_B) * g.ring_n_q != g.M))
    MLA_FAIL(MLA_ERR_INVALID_ARG, "GEMM ring epilogue: inconsistent ring geometry");
  if (g.rk != nullptr &&
      (g.batch != 1 || g.rk_col % 32 != 0 || g.rk_col < 0 || g.rk_col + g.rk_dr > g.N ||
       (g.rk_dr != 16 && g.rk_dr != 32 && g.rk_dr != 64) || g.rk_dr != 2 * (g.rope.pt + g.rope.ph + g.rope.pw) ||
       g.rk_D != g.rk_dc + g.rk_dr || g.rk_n_q <= 0 || g.rk_n_q % g.rope.tpf != 0 ||
       static_cast<int64_t>(g.rk_B) * g.rk_n_q != g.M || g.rk_nc_pad < g.rk_nc ||
       g.rk_rows < g.rk_nc_pad + g.rk_n_q || (g.rk_ring && g.rk_nc > 0 && g.rk_cache == nullptr) ||
       g.rk_slot_frame == nullptr || (reinterpret_cast<uintptr_t>(g.rk) & 15u) != 0 ||
       (g.rk_cache != nullptr && (reinterpret_cast<uintptr_t>(g.rk_cache) & 15u) != 0) ||
       (g.rk_D * 2) % 16 != 0 || (g.rk_dc * 2) % 16 != 0 ||
       static_cast<int64_t>(g.rk_B) * g.rk_rows >= (int64_t{1} << 31)))
    MLA_FAIL(MLA_ERR_INVALID_ARG, "GEMM rotated-key epilogue: inconsistent key geometry");
  if (g.epilogue == kEpiRopeQ &&
      (g.rope_D <= 0 || g.N % g.rope_D != 0 || g.rope_dr % 2 != 0 || g.rope_dr > g.rope_D ||
       g.rope_dr / 2 > kMaxRopePairs))
    MLA_FAIL(MLA_ERR_UNSUPPORTED, "query RoPE epilogue needs whole head blocks and even d_rope");
  // Tile width: the one with the least modelled time.  A persistent CTA takes ceil(tiles / SMs)
  // tiles one after another, and a tile's main loop is paced by the operand bytes it streams
  // into shared memory, K * (128 + width) * 2 (measured: these GEMMs run far below the tensor
  // rate), so the model is rounds * (128 + width); ties go to the wider tile.  Few rows (one
  // chunk) favour a width that fills every SM in one round; many rows favour wide tiles, which
  // re-read the A panel fewer times (x-projection of 32 chunks: 263 us with 256-wide tiles
  // against 728 us with 64-wide ones, which an SM-fill criterion alone had picked).
  const int sms = num_sms();
  const int widths[5] = {256, 224, 192, 128, 64};
  int best = 256;
  long long best_cost = -1;
  for (int w : widths) {
    const long long tiles =
        static_cast<long long>(ceil_div(g.M, kBM)) * ceil_div(g.N, w) * g.batch;
    const long long rounds = (tiles + sms - 1) / sms;
    const long long cost = rounds * (kBM + w);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = w;
    }
  }
  switch (best) {
    case 64: return launch_gemm<64>(g, s);
    case 128: return launch_gemm<128>(g, s);
    case 192: return launch_gemm<192>(g, s);
    case 224: return launch_gemm<224>(g, s);
    default: return launch_gemm<256>(g, s);
  }
}

}  // namespace mla
