// attention_bwd_sm100.cu - the attention backward on the sm_100a tensor cores, for the Wan latent
// shape (d_c 192, d_rope 32: D 224).  Same mathematics as attention_bwd.cu (see there); here the
// products are tcgen05 MMAs with fp32 accumulators in TMEM and bf16 operands (P and dS are
// rounded to bf16 as MMA operands; the softmax statistics stay fp32).
//
// dQ kernel: one CTA per (128-row query tile, head, sample); the key tiles stream through a
// 2-stage ring.  Per key tile j:
//   S   = Q' K'_j^T        M128 N128 K224   (A: Q' smem, B: K'_j smem, both K-major)
//   dP  = G  V_j^T         M128 N128 K192   (A: G smem, B: content blocks of K'_j, K-major)
//   dS  = scale * P o (dP - Delta), P = exp(S scale - lse)  (softmax warps, bf16 into TMEM)
//   dQ += dS K'_j          M128 N192 + N32  K128 (A: dS in TMEM, B: K'_j read MN-major)
// Key kernel: one CTA per (128-key tile, group of heads, sample); for every (head, query tile)
// of its group:
//   S^T  = K' Q'^T         M128 N128 K224
//   dP^T = V G^T           M128 N128 K192
//   P^T, dS^T (scaled)     softmax warps, one key row per thread, lse/Delta per query column
//   dL  += P^T G           M128 N192 K128   (value gradient: the value is the content latent)
//   dL  += dS^T Q'         M128 N192 + N32 K128 (key gradient, content and positional parts)
// dL (fp32, 224 wide) goes to a workspace slice per head group; bwd_reduce_kernel sums the
// groups, maps the positional part back through the transposed rotation and stores bf16.
// TMEM columns: S [0,128), dP [128,256), accumulator [256,480); P^T / dS are written over the
// first 64 columns of S and of dP.  Roles (192 threads): warps 0-3 softmax and epilogue (one
// TMEM lane = one row), warp 4 TMA producer, warp 5 TMEM allocation and the MMA thread.  Every
// wait is bounded; a wait that runs out writes MLA_ERR_DEVICE_TIMEOUT to dev_status.
#include "kernels.h"
#include "sm100.cuh"

namespace mla {

namespace {

using namespace sm100;

constexpr int kR = 128;                     // rows of every tile (queries or keys)
constexpr int kDc = 192, kDr = 32, kD = 224;
constexpr int kBlk = kR * 128;              // 16 KB: 128 rows x 128 B (64 bf16), 128B swizzle
constexpr int kRopeBlk = kR * 64;           // 8 KB: 128 rows x 64 B (32 bf16), 64B swizzle
constexpr int kTileD = 3 * kBlk + kRopeBlk; // 56 KB: a 128 x 224 tile (Q' or K')
constexpr int kTileG = 3 * kBlk;            // 48 KB: a 128 x 192 tile (G)
constexpr uint32_t kColS = 0, kColDP = 128, kColAcc = 256;
constexpr uint32_t kTmemCols = 512;
constexpr int kThreads = 192;
constexpr int kProducerWarp = 4, kMmaWarp = 5;
constexpr int kSoftmaxThreads = 128;
constexpr int kQStages = 2;                 // dQ kernel: K' ring
constexpr int kSmemQ = kTileD + kTileG + kQStages * kTileD + 1024;
constexpr int kStats = 2 * kR * 4;          // lse and Delta of a query tile: 1 KB
constexpr int kSmemK = kTileD + kTileD + kTileG + kStats + 1024;   // K' + one (Q', G) stage
constexpr float kLog2e = 1.4426950408889634f;

struct BwdTcParams {
  int n_q, H, nc, nc_pad, nt_ring, nt, rows_ws, heads_per_group, n_qt;
  float scale, scale_log2;
  const float* lse;      // [B, H, n_q]
  const float* delta;    // [B, H, n_q]
  void* d_q;             // [B, n_q, H, D] bf16
  float* partial;        // [groups, B, rows_ws, D] fp32
  int32_t* dev_status;
};

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// K-major tile operand (content blocks, 128B swizzle) and its positional block (64B swizzle).
__device__ __forceinline__ uint64_t kmajor_content(uint32_t a) {
  return smem_desc(a, 16, 1024, kSwizzle128B);
}
__device__ __forceinline__ uint64_t kmajor_rope(uint32_t a) {
  return smem_desc(a, 16, 512, kSwizzle64B);
}
// The same blocks read MN-major (N = columns of the tile, K = its rows): atoms of 64 (resp. 32)
// columns x 8 rows; LBO = stride between column blocks, SBO = stride between 8-row groups.
__device__ __forceinline__ uint64_t mnmajor_content(uint32_t a) {
  return smem_desc(a, kBlk, 1024, kSwizzle128B);
}
__device__ __forceinline__ uint64_t mnmajor_rope(uint32_t a) {
  return smem_desc(a, kRopeBlk, 512, kSwizzle64B);
}

constexpr uint32_t kIdescNN = idesc_bf16_f32(kR, 128, 0, 0);   // S, dP (both K-major)
constexpr uint32_t kIdescC = idesc_bf16_f32(kR, kDc, 0, 1);    // A TMEM, B MN-major, N 192
constexpr uint32_t kIdescR = idesc_bf16_f32(kR, kDr, 0, 1);    // A TMEM, B MN-major, N 32
constexpr uint32_t kBlkD = kBlk >> 4;

// D = A B^T over a 224-wide K (12 content k-steps + 2 positional ones); A, B tile bases.
__device__ __forceinline__ void mma_k224(uint32_t d, uint32_t a_tile, uint32_t b_tile) {
  const uint64_t ac = kmajor_content(a_tile), bc = kmajor_content(b_tile);
  const uint64_t ar = kmajor_rope(a_tile + 3 * kBlk), br = kmajor_rope(b_tile + 3 * kBlk);
#pragma unroll
  for (int blk = 0; blk < 3; ++blk)
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_ss(d, ac + (blk * kBlkD + 2 * kk), bc + (blk * kBlkD + 2 * kk), kIdescNN,
             (blk | kk) != 0 ? 1u : 0u);
#pragma unroll
  for (int kk = 0; kk < 2; ++kk) mma_ss(d, ar + 2 * kk, br + 2 * kk, kIdescNN, 1u);
}

// D = A B^T over the 192 content columns only.
__device__ __forceinline__ void mma_k192(uint32_t d, uint32_t a_tile, uint32_t b_tile) {
  const uint64_t ac = kmajor_content(a_tile), bc = kmajor_content(b_tile);
#pragma unroll
  for (int blk = 0; blk < 3; ++blk)
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_ss(d, ac + (blk * kBlkD + 2 * kk), bc + (blk * kBlkD + 2 * kk), kIdescNN,
             (blk | kk) != 0 ? 1u : 0u);
}

// acc[:, 0:192] (+)= A_tmem (128 x 128, bf16) . tile[:, 0:192]; with_rope: also
// acc[:, 192:224] (+)= A_tmem . tile[:, 192:224].  K = the tile's 128 rows.
__device__ __forceinline__ void mma_tmem_by_tile(uint32_t acc, uint32_t a_tmem, uint32_t tile,
                                                 bool with_rope, bool accumulate) {
  const uint64_t bc = mnmajor_content(tile);
  const uint64_t br = mnmajor_rope(tile + 3 * kBlk);
#pragma unroll
  for (int kk = 0; kk < kR / 16; ++kk) {
    // 16 rows further per k-step: 2048 B (content, 128 B rows) and 1024 B (rope, 64 B rows)
    mma_ts(acc, a_tmem + kk * 8, bc + 128 * kk, kIdescC, (accumulate || kk) ? 1u : 0u);
    if (with_rope)
      mma_ts(acc + kDc, a_tmem + kk * 8, br + 64 * kk, kIdescR, (accumulate || kk) ? 1u : 0u);
  }
}

// -------------------------------------------------------------------------------- dQ kernel

__global__ void __launch_bounds__(kThreads, 1)
    bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_qr,
                     const __grid_constant__ CUtensorMap tm_g,
                     const __grid_constant__ CUtensorMap tm_cache,
                     const __grid_constant__ CUtensorMap tm_chunk,
                     const __grid_constant__ CUtensorMap tm_ws, BwdTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t qg_full;
  __shared__ __align__(8) uint64_t kv_full[kQStages];
  __shared__ __align__(8) uint64_t kv_empty[kQStages];
  __shared__ __align__(8) uint64_t s_full;       // S and dP of tile j are in TMEM
  __shared__ __align__(8) uint64_t ds_full;      // the softmax has written dS(j)
  __shared__ __align__(8) uint64_t dq_done;      // the dQ products of tile j have completed
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sQ = sbase, sG = sbase + kTileD, sK = sbase + kTileD + kTileG;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int q0 = qt * kR;
  volatile int* abort_flag = &abort_sh;

  if (threadIdx.x == 0) {
    abort_sh = 0;
    mbar_init(smem_u32(&qg_full), 1);
    for (int s = 0; s < kQStages; ++s) {
      mbar_init(smem_u32(&kv_full[s]), 1);
      mbar_init(smem_u32(&kv_empty[s]), 1);
    }
    mbar_init(smem_u32(&s_full), 1);
    mbar_init(smem_u32(&ds_full), kSoftmaxThreads);
    mbar_init(smem_u32(&dq_done), 1);
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(&tmem_base_sh), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp == kProducerWarp) {
    if (lane == 0) {
      const uint32_t qb = smem_u32(&qg_full);
      mbar_arrive_expect_tx(qb, kTileD + kTileG);
      for (int i = 0; i < 3; ++i) tma_load_4d(sQ + i * kBlk, &tm_q, qb, 64 * i, h, q0, b);
      tma_load_4d(sQ + 3 * kBlk, &tm_qr, qb, kDc, h, q0, b);
      for (int i = 0; i < 3; ++i) tma_load_4d(sG + i * kBlk, &tm_g, qb, 64 * i, h, q0, b);
      bool ok = true;
      for (int j = 0; j < p.nt && ok; ++j) {
        const int s = j % kQStages;
        ok = mbar_wait_or_abort(smem_u32(&kv_empty[s]), ((j / kQStages) & 1) ^ 1, abort_flag,
                                p.dev_status);
        if (!ok) break;
        const uint32_t dst = sK + s * kTileD;
        const uint32_t fb = smem_u32(&kv_full[s]);
        mbar_arrive_expect_tx(fb, kTileD);
        if (j < p.nt_ring) {
          const int r0 = j * kR;
          for (int i = 0; i < 3; ++i) tma_load_3d(dst + i * kBlk, &tm_cache, fb, 64 * i, r0, b);
          tma_load_3d(dst + 3 * kBlk, &tm_ws, fb, 0, r0, b);
        } else {
          const int r0 = (j - p.nt_ring) * kR;
          for (int i = 0; i < 3; ++i) tma_load_3d(dst + i * kBlk, &tm_chunk, fb, 64 * i, r0, b);
          tma_load_3d(dst + 3 * kBlk, &tm_ws, fb, 0, p.nc_pad + r0, b);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      bool ok = mbar_wait_or_abort(smem_u32(&qg_full), 0, abort_flag, p.dev_status);
      for (int j = 0; j < p.nt && ok; ++j) {
        const int s = j % kQStages;
        ok = mbar_wait_or_abort(smem_u32(&kv_full[s]), (j / kQStages) & 1, abort_flag,
                                p.dev_status);
        // dS(j-1) sits in the S columns: its dQ products must have read it
        if (ok && j > 0)
          ok = mbar_wait_or_abort(smem_u32(&dq_done), (j - 1) & 1, abort_flag, p.dev_status);
        if (!ok) break;
        tc_fence_after();
        const uint32_t kt = sK + s * kTileD;
        mma_k224(tmem + kColS, sQ, kt);
        mma_k192(tmem + kColDP, sG, kt);
        mma_commit(smem_u32(&s_full));
        ok = mbar_wait_or_abort(smem_u32(&ds_full), j & 1, abort_flag, p.dev_status);
        if (!ok) break;
        tc_fence_after();
        mma_tmem_by_tile(tmem + kColAcc, tmem + kColS, kt, true, j > 0);
        mma_commit(smem_u32(&kv_empty[s]));
        mma_commit(smem_u32(&dq_done));
      }
    }
  } else {
    // softmax warps: one query row per thread
    const int row = warp * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const int n = q0 + row;
    const bool row_ok = n < p.n_q;
    const int64_t sr = (static_cast<int64_t>(b) * p.H + h) * p.n_q + n;
    const float lse2 = row_ok ? p.lse[sr] * kLog2e : INFINITY;   // invalid rows: p = 0
    const float delta = row_ok ? p.delta[sr] : 0.f;
    bool ok = true;
    for (int j = 0; j < p.nt && ok; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait_or_abort(smem_u32(&s_full), j & 1, abort_flag,
                                                      p.dev_status));
      if (!ok) break;
      tc_fence_after();
      const int valid = j < p.nt_ring ? min(kR, p.nc - j * kR)
                                      : min(kR, p.n_q - (j - p.nt_ring) * kR);
      // two halves of 64 keys; dS of half k goes to S columns [32k, 32k + 32), which hold
      // scores that have been read already
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        uint32_t rs[64], rp[64];
        tmem_ld64_wait(tmem + lane_off + kColS + 64 * half, rs);
        tmem_ld64_wait(tmem + lane_off + kColDP + 64 * half, rp);
        uint32_t w[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          float d2[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int c = 2 * i + u;
            const float pr = 64 * half + c < valid
                ? fast_exp2(__uint_as_float(rs[c]) * p.scale_log2 - lse2) : 0.f;
            d2[u] = pr * (__uint_as_float(rp[c]) - delta) * p.scale;
          }
          w[i] = pack_bf16x2(d2[0], d2[1]);
        }
#pragma unroll
        for (int c = 0; c < 32; c += 16) {
          uint32_t w16[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) w16[i] = w[c + i];
          tmem_st16(tmem + lane_off + kColS + 32 * half + c, w16);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&ds_full));
    }
    if (ok)
      ok = __all_sync(0xffffffffu, mbar_wait_or_abort(smem_u32(&dq_done), (p.nt - 1) & 1,
                                                      abort_flag, p.dev_status));
    if (ok) {
      tc_fence_after();
      bf16* out = static_cast<bf16*>(p.d_q) + ((static_cast<int64_t>(b) * p.n_q + n) * p.H + h) * kD;
#pragma unroll 1
      for (int c = 0; c < kD; c += 32) {
        uint32_t r[32];
        tmem_ld32_wait(tmem + lane_off + kColAcc + c, r);
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) w[i] = pack_bf16x2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
        if (row_ok) {
          uint4* d4 = reinterpret_cast<uint4*>(out + c);
#pragma unroll
          for (int i = 0; i < 4; ++i) d4[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------------------- key kernel

__global__ void __launch_bounds__(kThreads, 1)
    bwd_dkey_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_qr,
                       const __grid_constant__ CUtensorMap tm_g,
                       const __grid_constant__ CUtensorMap tm_cache,
                       const __grid_constant__ CUtensorMap tm_chunk,
                       const __grid_constant__ CUtensorMap tm_ws, BwdTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t k_full;
  __shared__ __align__(8) uint64_t qg_full;     // Q'(i), G(i) landed
  __shared__ __align__(8) uint64_t qg_empty;    // the products of iteration i have read them
  __shared__ __align__(8) uint64_t s_full;
  __shared__ __align__(8) uint64_t ps_full;
  __shared__ __align__(8) uint64_t acc_done;    // the dL products of iteration i completed
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sK = sbase, sQ = sbase + kTileD, sG = sbase + 2 * kTileD;
  const uint32_t sStats = sG + kTileG;          // lse [128] then Delta [128] of the query tile
  const float* col_lse = reinterpret_cast<const float*>(smem_raw + (sStats - smem_u32(smem_raw)));
  const float* col_delta = col_lse + kR;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int kt = blockIdx.x, grp = blockIdx.y, b = blockIdx.z;
  const int n_iter = p.heads_per_group * p.n_qt;
  volatile int* abort_flag = &abort_sh;

  if (threadIdx.x == 0) {
    abort_sh = 0;
    mbar_init(smem_u32(&k_full), 1);
    mbar_init(smem_u32(&qg_full), 1);
    mbar_init(smem_u32(&qg_empty), 1);
    mbar_init(smem_u32(&s_full), 1);
    mbar_init(smem_u32(&ps_full), kSoftmaxThreads);
    mbar_init(smem_u32(&acc_done), 1);
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(&tmem_base_sh), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp == kProducerWarp) {
    if (lane == 0) {
      const uint32_t kb = smem_u32(&k_full);
      mbar_arrive_expect_tx(kb, kTileD);
      if (kt < p.nt_ring) {
        const int r0 = kt * kR;
        for (int i = 0; i < 3; ++i) tma_load_3d(sK + i * kBlk, &tm_cache, kb, 64 * i, r0, b);
        tma_load_3d(sK + 3 * kBlk, &tm_ws, kb, 0, r0, b);
      } else {
        const int r0 = (kt - p.nt_ring) * kR;
        for (int i = 0; i < 3; ++i) tma_load_3d(sK + i * kBlk, &tm_chunk, kb, 64 * i, r0, b);
        tma_load_3d(sK + 3 * kBlk, &tm_ws, kb, 0, p.nc_pad + r0, b);
      }
      bool ok = true;
      for (int it = 0; it < n_iter && ok; ++it) {
        ok = mbar_wait_or_abort(smem_u32(&qg_empty), (it & 1) ^ 1, abort_flag, p.dev_status);
        if (!ok) break;
        const int h = grp * p.heads_per_group + it / p.n_qt;
        const int q0 = (it % p.n_qt) * kR;
        // column statistics of the query tile: n_q is a multiple of 4, so both the source
        // (row (b, h) of [B, H, n_q] floats, column q0) and the size are 16-byte multiples
        const uint32_t stat_bytes = static_cast<uint32_t>(min(kR, p.n_q - q0)) * 4u;
        const int64_t so = (static_cast<int64_t>(b) * p.H + h) * p.n_q + q0;
        const uint32_t fb = smem_u32(&qg_full);
        mbar_arrive_expect_tx(fb, kTileD + kTileG + 2 * stat_bytes);
        for (int i = 0; i < 3; ++i) tma_load_4d(sQ + i * kBlk, &tm_q, fb, 64 * i, h, q0, b);
        tma_load_4d(sQ + 3 * kBlk, &tm_qr, fb, kDc, h, q0, b);
        for (int i = 0; i < 3; ++i) tma_load_4d(sG + i * kBlk, &tm_g, fb, 64 * i, h, q0, b);
        bulk_load(sStats, p.lse + so, stat_bytes, fb);
        bulk_load(sStats + kR * 4, p.delta + so, stat_bytes, fb);
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      bool ok = mbar_wait_or_abort(smem_u32(&k_full), 0, abort_flag, p.dev_status);
      for (int it = 0; it < n_iter && ok; ++it) {
        ok = mbar_wait_or_abort(smem_u32(&qg_full), it & 1, abort_flag, p.dev_status);
        // P^T(it-1) and dS^T(it-1) sit in the S and dP columns until their products completed
        if (ok && it > 0)
          ok = mbar_wait_or_abort(smem_u32(&acc_done), (it - 1) & 1, abort_flag, p.dev_status);
        if (!ok) break;
        tc_fence_after();
        mma_k224(tmem + kColS, sK, sQ);
        mma_k192(tmem + kColDP, sK, sG);
        mma_commit(smem_u32(&s_full));
        ok = mbar_wait_or_abort(smem_u32(&ps_full), it & 1, abort_flag, p.dev_status);
        if (!ok) break;
        tc_fence_after();
        // value gradient P^T G into the content columns, then the key gradient dS^T Q'
        // (the positional accumulator columns get no value term; the softmax warps zeroed them
        // before their first arrival, so every product into them accumulates)
        mma_tmem_by_tile(tmem + kColAcc, tmem + kColS, sG, false, it > 0);
        mma_tmem_by_tile(tmem + kColAcc, tmem + kColDP, sQ, true, true);
        mma_commit(smem_u32(&qg_empty));
        mma_commit(smem_u32(&acc_done));
      }
    }
  } else {
    const int row = warp * 32 + lane;           // key row of the tile
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const bool key_ok = kt < p.nt_ring ? kt * kR + row < p.nc
                                       : (kt - p.nt_ring) * kR + row < p.n_q;
    // the positional accumulator columns have no value term: zero them before any product
    {
      uint32_t z[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) z[i] = 0u;
      tmem_st16(tmem + lane_off + kColAcc + kDc, z);
      tmem_st16(tmem + lane_off + kColAcc + kDc + 16, z);
      tmem_wait_st();
    }
    bool ok = true;
    for (int it = 0; it < n_iter && ok; ++it) {
      // S^T(it) and dP^T(it), and the column statistics that the bulk copies of qg_full(it)
      // brought (observed directly: the copies complete on that barrier)
      ok = __all_sync(0xffffffffu,
                      mbar_wait_or_abort(smem_u32(&s_full), it & 1, abort_flag, p.dev_status) &&
                          mbar_wait_or_abort(smem_u32(&qg_full), it & 1, abort_flag, p.dev_status));
      if (!ok) break;
      tc_fence_after();
      const int q0 = (it % p.n_qt) * kR;
      const int ncols = min(kR, p.n_q - q0);
      // two halves of 64 query columns; P^T / dS^T of half k go to columns [32k, 32k + 32) of
      // S / dP, which hold values that have been read already
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        uint32_t rs[64], rp[64];
        tmem_ld64_wait(tmem + lane_off + kColS + 64 * half, rs);
        tmem_ld64_wait(tmem + lane_off + kColDP + 64 * half, rp);
        uint32_t wp[32], wd[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          float pp[2], dd[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int c = 64 * half + 2 * i + u;
            const bool col_ok = key_ok && c < ncols;
            const float pr = col_ok ? fast_exp2(__uint_as_float(rs[2 * i + u]) * p.scale_log2 -
                                                col_lse[c] * kLog2e)
                                    : 0.f;
            pp[u] = pr;
            dd[u] = col_ok ? pr * (__uint_as_float(rp[2 * i + u]) - col_delta[c]) * p.scale : 0.f;
          }
          wp[i] = pack_bf16x2(pp[0], pp[1]);
          wd[i] = pack_bf16x2(dd[0], dd[1]);
        }
#pragma unroll
        for (int c = 0; c < 32; c += 16) {
          uint32_t w16[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) w16[i] = wp[c + i];
          tmem_st16(tmem + lane_off + kColS + 32 * half + c, w16);
#pragma unroll
          for (int i = 0; i < 16; ++i) w16[i] = wd[c + i];
          tmem_st16(tmem + lane_off + kColDP + 32 * half + c, w16);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&ps_full));
    }
    if (ok)
      ok = __all_sync(0xffffffffu, mbar_wait_or_abort(smem_u32(&acc_done), (n_iter - 1) & 1,
                                                      abort_flag, p.dev_status));
    if (ok) {
      tc_fence_after();
      const int prow = kt < p.nt_ring ? kt * kR + row : p.nc_pad + (kt - p.nt_ring) * kR + row;
      float* out = p.partial +
                   ((static_cast<int64_t>(grp) * gridDim.z + b) * p.rows_ws + prow) * kD;
#pragma unroll 1
      for (int c = 0; c < kD; c += 32) {
        uint32_t r[32];
        tmem_ld32_wait(tmem + lane_off + kColAcc + c, r);
        float4* d4 = reinterpret_cast<float4*>(out + c);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          d4[i] = make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                              __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Sums the head groups' partial latent gradients of every attended key, maps the positional
// part back through the transposed rotation and stores bf16 into d_cache / d_chunk_lat.
__global__ void bwd_reduce_kernel(const float* __restrict__ partial, int groups, int B,
                                  int rows_ws, int nc, int nc_pad, int n_q, int W, int tpf,
                                  int frame_w, int first_frame, const int32_t* slot_frame,
                                  RopeGeom g, bf16* d_cache, bf16* d_chunk_lat) {
  const int nk = nc + n_q;
  const int64_t total = static_cast<int64_t>(B) * nk * (kD / 2);   // one pair per thread
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int pr = static_cast<int>(e % (kD / 2));
    const int64_t bm = e / (kD / 2);
    const int m = static_cast<int>(bm % nk), b = static_cast<int>(bm / nk);
    const int prow = m < nc ? m : nc_pad + (m - nc);
    float x0 = 0.f, x1 = 0.f;
    for (int gi = 0; gi < groups; ++gi) {
      const float* src = partial + ((static_cast<int64_t>(gi) * B + b) * rows_ws + prow) * kD + 2 * pr;
      x0 += src[0];
      x1 += src[1];
    }
    if (2 * pr >= kDc) {
      int t, hh, ww;
      key_position(slot_frame, b, W, tpf, frame_w, nc, first_frame, m, t, hh, ww);
      rope_rotate(x0, x1, -rope_angle(g, (2 * pr - kDc) / 2, t, hh, ww));
    }
    bf16* dst = m < nc ? d_cache + (static_cast<int64_t>(b) * W * tpf + m) * kD
                       : d_chunk_lat + (static_cast<int64_t>(b) * n_q + (m - nc)) * kD;
    __nv_bfloat162 v = __floats2bfloat162_rn(x0, x1);
    *reinterpret_cast<__nv_bfloat162*>(dst + 2 * pr) = v;
  }
}

}  // namespace

int bwd_tc_head_groups(const Dims& d, int n_valid) {
  // The key kernel has one CTA per (key tile, head group, sample); pick the number of head
  // groups (a divisor of H) whose CTAs fill whole waves of 148 SMs best, the fewest on ties
  // (each group adds a partial gradient to sum and re-reads the key tile).
  const KeyWorkspace k = key_workspace_layout(d, n_valid);
  const long long tiles = static_cast<long long>(ceil_div(k.nc, kR) + ceil_div(d.n_q, kR)) * d.B;
  int best = 1;
  double best_eff = -1.0;
  for (int g = 1; g <= d.H; ++g) {
    if (d.H % g != 0) continue;
    const long long ctas = tiles * g;
    const double eff = static_cast<double>(ctas) / (((ctas + 147) / 148) * 148.0);
    if (eff > best_eff + 1e-9) {
      best_eff = eff;
      best = g;
    }
  }
  return best;
}

bool tc_bwd_supported(const Dims& d) {
  // n_q a multiple of 4: the key kernel copies a query tile's lse / Delta with 16-byte bulk copies
  return d.dtype == MLA_BF16 && d.path == MLA_PATH_AUTO && d.d_c == kDc && d.d_rope == kDr &&
         d.n_q % 4 == 0;
}

mla_status attention_bwd_tc(const Dims& d, const BwdArgs& a, int n_valid, int first_frame,
                            const float* delta, const void* ws_rope, float* partial, int groups,
                            int32_t* dev_status, cudaStream_t s) {
  const KeyWorkspace kw = key_workspace_layout(d, n_valid);
  CUtensorMap tq, tqr, tg, tcache, tchunk, tws;
  mla_status st;
  {
    const uint64_t dims[4] = {static_cast<uint64_t>(kD), static_cast<uint64_t>(d.H),
                              static_cast<uint64_t>(d.n_q), static_cast<uint64_t>(d.B)};
    const uint64_t strides[3] = {kD * 2ull, static_cast<uint64_t>(d.H) * kD * 2,
                                 static_cast<uint64_t>(d.n_q) * d.H * kD * 2};
    const uint32_t box[4] = {64, 1, kR, 1};
    if ((st = make_tmap_bf16(&tq, a.q, 4, dims, strides, box, 128)) != MLA_OK) return st;
    const uint32_t box_r[4] = {kDr, 1, kR, 1};
    if ((st = make_tmap_bf16(&tqr, a.q, 4, dims, strides, box_r, 64)) != MLA_OK) return st;
  }
  {
    const uint64_t dims[4] = {static_cast<uint64_t>(kDc), static_cast<uint64_t>(d.H),
                              static_cast<uint64_t>(d.n_q), static_cast<uint64_t>(d.B)};
    const uint64_t strides[3] = {kDc * 2ull, static_cast<uint64_t>(d.H) * kDc * 2,
                                 static_cast<uint64_t>(d.n_q) * d.H * kDc * 2};
    const uint32_t box[4] = {64, 1, kR, 1};
    if ((st = make_tmap_bf16(&tg, a.d_o_lat, 4, dims, strides, box, 128)) != MLA_OK) return st;
  }
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(kD), static_cast<uint64_t>(d.n_q),
                              static_cast<uint64_t>(d.B)};
    const uint64_t strides[2] = {kD * 2ull, static_cast<uint64_t>(d.n_q) * kD * 2};
    const uint32_t box[3] = {64, kR, 1};
    if ((st = make_tmap_bf16(&tchunk, a.chunk_lat, 3, dims, strides, box, 128)) != MLA_OK) return st;
  }
  if (kw.nc > 0) {
    const uint64_t dims[3] = {static_cast<uint64_t>(kD), static_cast<uint64_t>(kw.nc),
                              static_cast<uint64_t>(d.B)};
    const uint64_t strides[2] = {kD * 2ull, static_cast<uint64_t>(d.W) * d.tpf * kD * 2};
    const uint32_t box[3] = {64, kR, 1};
    if ((st = make_tmap_bf16(&tcache, a.cache, 3, dims, strides, box, 128)) != MLA_OK) return st;
  } else {
    tcache = tchunk;
  }
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(kDr), static_cast<uint64_t>(kw.rows),
                              static_cast<uint64_t>(d.B)};
    const uint64_t strides[2] = {kDr * 2ull, static_cast<uint64_t>(kw.rows) * kDr * 2};
    const uint32_t box[3] = {kDr, kR, 1};
    if ((st = make_tmap_bf16(&tws, ws_rope, 3, dims, strides, box, 64)) != MLA_OK) return st;
  }
  BwdTcParams p;
  p.n_q = d.n_q; p.H = d.H; p.nc = kw.nc; p.nc_pad = kw.nc_pad;
  p.nt_ring = ceil_div(kw.nc, kR);
  p.nt = p.nt_ring + ceil_div(d.n_q, kR);
  p.rows_ws = kw.rows; p.heads_per_group = d.H / groups; p.n_qt = ceil_div(d.n_q, kR);
  p.scale = d.scale; p.scale_log2 = d.scale * kLog2e;
  p.lse = a.lse; p.delta = delta; p.d_q = a.d_q; p.partial = partial; p.dev_status = dev_status;
  MLA_CUDA_TRY(cudaFuncSetAttribute(bwd_dq_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    kSmemQ));
  MLA_CUDA_TRY(cudaFuncSetAttribute(bwd_dkey_tc_kernel,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemK));
  dim3 gq(ceil_div(d.n_q, kR), d.H, d.B);
  bwd_dq_tc_kernel<<<gq, kThreads, kSmemQ, s>>>(tq, tqr, tg, tcache, tchunk, tws, p);
  MLA_LAUNCH_CHECK("bwd_dq_tc");
  dim3 gk(p.nt, groups, d.B);
  bwd_dkey_tc_kernel<<<gk, kThreads, kSmemK, s>>>(tq, tqr, tg, tcache, tchunk, tws, p);
  MLA_LAUNCH_CHECK("bwd_dkey_tc");
  const int64_t total = static_cast<int64_t>(d.B) * (kw.nc + d.n_q) * (kD / 2);
  const int blocks = static_cast<int>(std::min<int64_t>((total + 255) / 256, 148 * 16));
  bwd_reduce_kernel<<<blocks, 256, 0, s>>>(partial, groups, d.B, kw.rows, kw.nc, kw.nc_pad, d.n_q,
                                           d.W, d.tpf, d.frame_w, first_frame, a.slot_frame,
                                           rope_geom(d), static_cast<bf16*>(a.d_cache),
                                           static_cast<bf16*>(a.d_chunk_lat));
  MLA_LAUNCH_CHECK("bwd_reduce");
  return MLA_OK;
}

}  // namespace mla
