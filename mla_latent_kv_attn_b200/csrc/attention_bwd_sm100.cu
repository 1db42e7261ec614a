// attention_bwd_sm100.cu - the attention backward on the sm_100a tensor cores, for the Wan latent
// shape (d_c 192, d_rope 32: D 224).  Same mathematics as attention_bwd.cu (see there); here the
// products are tcgen05 MMAs with fp32 accumulators in TMEM and bf16 operands (P and dS are
// rounded to bf16 as MMA operands; the softmax statistics stay fp32).
//
// Both kernels own a 128-row tile and stream 64-row sub-tiles of the other side through a ring
// of shared-memory stages.  The operand a CTA keeps for its whole life (its 128 query rows Q' in
// the dQ kernel, its 128 keys K' in the key kernel) sits in TMEM as bf16 pairs, so the S and dP
// MMAs read only their streamed B operand from shared memory.  (Measured on this part: an M128
// K16 MMA with N <= 64 costs ~45 cycles with A in TMEM and ~48 with A in shared memory, against
// 32 cycles of work, whatever else is in flight; N = 128 and 256 run at the full rate.  Hence the
// key kernel computes S and dP as one N=128 product, below.)  The softmax warps load S and dP
// into registers and release the TMEM buffers at once, so the S/dP MMAs of the next sub-tile
// overlap the softmax; P and dS go to
// shared memory (128-byte-swizzled K-major rows, written the way a TMA load would place them)
// as the A operands of the key kernel's gradient products; the dQ kernel keeps dS in TMEM,
// in the 32 columns its N=224 accumulator leaves free.
// A streamed sub-tile that is read MN-major (K'_j in the dQ kernel, Q'_i in the key kernel) is
// held 256 columns wide: three 64-column content blocks and a fourth block with the 32
// positional columns followed by 32 zeros, all with the 128-byte swizzle. Its product is then a
// single MMA per k-step instead of an N=192 and a separate, slow, N=32 one: N=256 in the key
// kernel (columns 224-255 of its accumulator receive zeros and are never read), N=224 in the
// dQ kernel (the zero half of the fourth block is not read). The keys come from a copy the
// pre-pass bwd_pad_keys_kernel assembles in the workspace; Q'_i's fourth block is a TMA box that
// runs past the query's 224 columns, which the copy engine fills with zeros.
// dQ kernel: one CTA per (128-row query tile, head, sample); per 64-key sub-tile j:
//   S_j  = Q' K'_j^T       M128 N64 K224    (A: Q' in TMEM, B: K'_j smem, K-major)
//   dP_j = G  V_j^T        M128 N64 K192    (A: G smem, B: content blocks of K'_j, K-major)
//   dS_j = scale * P o (dP - Delta), P = exp(S scale - lse)    (softmax warps, bf16 to TMEM)
//   dQ  += dS_j K'_j       M128 N224 K64    (A: dS in TMEM, B: K'_j read MN-major)
// Key kernel: one CTA per (128-key tile, group of heads, sample); per (head, 64-query sub-tile):
//   [S^T | dP^T] = K' [Q'_i ; G_i 0]^T   M128 N128 K224 (A: K' in TMEM; B: the stage stacks the
//                          Q' sub-tile over G with zeros in its positional columns, so the second
//                          half is V G_i^T)
//   P^T, scale * dS^T      softmax warps, one half key row per thread, lse/Delta per column
//   dL  += dS^T Q'_i       M128 N256 K64    (key gradient, content and positional parts)
//   dL  += P^T G_i         M128 N192 K64    (value gradient: the value is the content latent)
// dL (fp32, 224 wide) goes to a workspace slice per head group; bwd_reduce_kernel sums the
// groups, maps the positional part back through the transposed rotation and stores bf16.
// TMEM columns: resident A operand [0,112), S [128,192), dP [192,256), accumulator [256,512)
// (dQ kernel: [256,480), then dS [480,512)).
// Roles: softmax / epilogue warps (one TMEM lane = one row), a TMA producer warp, and a warp that
// allocates TMEM and whose lane 0 issues every MMA.  Every wait is bounded; a wait that runs out
// writes MLA_ERR_DEVICE_TIMEOUT to dev_status.
#include "exp2.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace mla {

namespace {

using namespace sm100;

constexpr int kR = 128;                     // rows of the tile a CTA owns
constexpr int kS = 64;                      // rows of a streamed sub-tile
constexpr int kDc = 192, kDr = 32, kD = 224;
constexpr int kBlkR = kR * 128;             // 16 KB: 128 rows x 128 B (64 bf16), 128B swizzle
constexpr int kBlkS = kS * 128;             // 8 KB:  64 rows x 128 B
constexpr int kTileGR = 3 * kBlkR;          // 48 KB: a 128 x 192 tile of G
constexpr int kTileS = 4 * kBlkS;           // 32 KB: a 64 x 256 sub-tile (rope block padded)
constexpr int kTileGS = 3 * kBlkS;          // 24 KB: a 64 x 192 sub-tile of G
constexpr int kOpBytes = kR * 128;          // 16 KB: a 128 x 64 bf16 operand (dS, P) in smem
constexpr uint32_t kColA = 0, kColS = 128, kColDP = 192, kColAcc = 256;
constexpr uint32_t kColDS = kColAcc + kD;   // dQ kernel: dS (bf16 pairs, 32 columns) after an
                                            // accumulator of N = 224
constexpr int kAWords = kD / 2;             // 112 TMEM columns of bf16 pairs
constexpr uint32_t kTmemCols = 512;
// dQ kernel: 4 softmax warps, producer, MMA
constexpr int kSoftmaxQ = 128, kThreadsQ = kSoftmaxQ + 64;
constexpr int kProducerWarpQ = 4, kMmaWarpQ = 5;
constexpr int kQStages = 5;                                   // K' sub-tiles in flight
constexpr int kSmemQ = kTileGR + kQStages * kTileS + 1024;
// key kernel: 8 softmax warps (two per TMEM lane quarter, each half of the columns)
constexpr int kSoftmaxK = 256, kThreadsK = kSoftmaxK + 64;
constexpr int kProducerWarpK = 8, kMmaWarpK = 9;
// a key-kernel stage stacks a Q' sub-tile over a G sub-tile: block i (64 columns) holds 128
// rows, Q' rows 0-63 then G rows 0-63; the G half of block 3 (past G's 192 columns) is zero
constexpr int kBlkQG = 2 * kBlkS;                             // 16 KB
constexpr int kKStage = 4 * kBlkQG;                           // 64 KB
constexpr int kKStages = 3;
constexpr int kStatBytes = 2 * kS * 4;                        // lse and Delta of a sub-tile
constexpr int kSmemK = kKStages * kKStage + 2 * kOpBytes + kKStages * kStatBytes + 1024;
static_assert(kSmemQ <= 227 * 1024 && kSmemK + 256 <= 227 * 1024, "shared memory");
constexpr float kLog2e = 1.4426950408889634f;

struct BwdTcParams {
  int n_q, H, nc, nc_pad, nt_ring, nt, rows_ws, heads_per_group;
  int ns_ring, ns;          // dQ kernel: 64-key sub-tiles of the ring, in all
  int n_qs;                 // key kernel: 64-query sub-tiles per head
  float scale, scale_log2;
  const bf16* q;         // [B, n_q, H, D]
  const bf16* keys;      // [B, rows_ws, 256] padded key copy
  const float* lse;      // [B, H, n_q]
  const float* delta;    // [B, H, n_q]
  void* d_q;             // [B, n_q, H, D] bf16
  float* partial;        // [groups, B, rows_ws, D] fp32
  int32_t* dev_status;
};

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

// 16-byte piece `chunk` (0-7) of row `row` of a K-major operand with 128-byte rows and the
// 128-byte swizzle (a 1024-byte-aligned buffer): the piece index is XORed with the row's position
// in its 8-row group, as a TMA load with that swizzle places it.
__device__ __forceinline__ uint32_t swz128(uint32_t buf, int row, int chunk) {
  return buf + static_cast<uint32_t>(row) * 128u + (static_cast<uint32_t>(chunk ^ (row & 7)) << 4);
}

// Descriptors of a tile's blocks.  K-major (rows = M or N, K = columns): 8-row atoms of 128-byte
// rows, SBO 1024.  MN-major (N = columns, K = rows): atoms of 64 columns x 8 rows; LBO = stride
// between column blocks, SBO = stride between 8-row groups.
__device__ __forceinline__ uint64_t kmajor_content(uint32_t a) {
  return smem_desc(a, 16, 1024, kSwizzle128B);
}
__device__ __forceinline__ uint64_t mnmajor_content(uint32_t a, uint32_t blk_bytes) {
  return smem_desc(a, blk_bytes, 1024, kSwizzle128B);
}

constexpr uint32_t kIdescS = idesc_bf16_f32(kR, kS, 0, 0);     // S, dP: M128 N64, K-major
constexpr uint32_t kIdescSD = idesc_bf16_f32(kR, 2 * kS, 0, 0); // [S | dP]: M128 N128, K-major
constexpr uint32_t kIdescC = idesc_bf16_f32(kR, kDc, 0, 1);    // B MN-major, N 192
constexpr uint32_t kIdescW = idesc_bf16_f32(kR, 256, 0, 1);    // B MN-major, N 256
constexpr uint32_t kIdescD = idesc_bf16_f32(kR, kD, 0, 1);     // B MN-major, N 224

// dQ kernel: S = Q' K'_j^T over K 224 (Q' in TMEM from column a_tmem) and dP = G V_j^T over the
// 192 content columns (G a K-major 128-row tile in shared memory, blocks kBlkR apart); K'_j a
// K-major 64-row sub-tile, blocks kBlkS apart.  Both are N=64 chains, at the ~45-cycle floor an
// M128 K16 instruction has for N <= 64 (32 cycles of work); their k-steps are issued alternately
// (a probe found no difference from issuing one chain after the other).
__device__ __forceinline__ void mma_s_dp(uint32_t s_acc, uint32_t dp_acc, uint32_t a_tmem,
                                         uint32_t g_smem, uint32_t k_tile) {
  const uint64_t bk = kmajor_content(k_tile), ag = kmajor_content(g_smem);
#pragma unroll
  for (int kk = 0; kk < kD / 16; ++kk) {
    const uint32_t off = (((kk >> 2) * kBlkS) >> 4) + 2 * (kk & 3);
    mma_ts(s_acc, a_tmem + 8 * kk, bk + off, kIdescS, kk ? 1u : 0u);
    if (kk < kDc / 16)
      mma_ss(dp_acc, ag + (((kk >> 2) * kBlkR) >> 4) + 2 * (kk & 3), bk + off, kIdescS,
             kk ? 1u : 0u);
  }
}

// [S | dP] = A [Q'_i ; G'_i]^T in one N=128 MMA chain over K 224: A (the key tile) in TMEM from
// column a_tmem, B a stacked stage (blocks kBlkQG apart).  G'_i is G_i with 32 zero columns
// appended, so the second half of the result is V G_i^T: the content columns of the key tile
// times G_i (the positional part meets the zeros).
__device__ __forceinline__ void mma_s_dp_stacked(uint32_t d, uint32_t a_tmem, uint32_t stage) {
  const uint64_t b = kmajor_content(stage);
#pragma unroll
  for (int kk = 0; kk < kD / 16; ++kk)
    mma_ts(d, a_tmem + 8 * kk, b + (((kk >> 2) * kBlkQG) >> 4) + 2 * (kk & 3), kIdescSD,
           kk ? 1u : 0u);
}

// acc[:, 0:kN] (+)= A (128 x 64 bf16, K-major 128-byte swizzled rows in smem) . sub[:, 0:kN],
// kN = 192 (content blocks) or 256 (all four blocks of a padded sub-tile), the sub-tile's
// 64-column blocks blk_bytes apart; K = its 64 rows, one MMA per k-step (A 32 bytes further, B
// 16 rows = 2048 bytes further).
template <int kN>
__device__ __forceinline__ void mma_op_by_sub(uint32_t acc, uint32_t a_smem, uint32_t sub,
                                              uint32_t blk_bytes, bool accumulate) {
  static_assert(kN == kDc || kN == 256, "product width");
  const uint64_t a = kmajor_content(a_smem);
  const uint64_t b = mnmajor_content(sub, blk_bytes);
#pragma unroll
  for (int kk = 0; kk < kS / 16; ++kk)
    mma_ss(acc, a + 2 * kk, b + 128 * kk, kN == kDc ? kIdescC : kIdescW,
           (accumulate || kk) ? 1u : 0u);
}

// acc[:, 0:224] (+)= A (128 x 64 bf16, pairs in TMEM from column a_tmem, 8 columns per k-step)
// . sub[:, 0:224], sub a padded sub-tile read MN-major (blocks kBlkS apart; the fourth block's
// zero half is not read).  K = its 64 rows.
__device__ __forceinline__ void mma_tmem_by_sub224(uint32_t acc, uint32_t a_tmem, uint32_t sub,
                                                   bool accumulate) {
  const uint64_t b = mnmajor_content(sub, kBlkS);
#pragma unroll
  for (int kk = 0; kk < kS / 16; ++kk)
    mma_ts(acc, a_tmem + 8 * kk, b + 128 * kk, kIdescD, (accumulate || kk) ? 1u : 0u);
}

// Writes `nwords` bf16 pairs of a global row (16-byte aligned; nullptr: zeros) into this thread's
// TMEM lane from column taddr on, 16 columns at a time.
__device__ __forceinline__ void row_to_tmem(uint32_t taddr, const bf16* src, int nwords) {
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
  for (int c = 0; c < nwords; c += 16) {
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 v = src != nullptr ? s4[c / 4 + i] : make_uint4(0u, 0u, 0u, 0u);
      w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
    }
    tmem_st16(taddr + c, w);
  }
}

// -------------------------------------------------------------------------------- dQ kernel

__global__ void __launch_bounds__(kThreadsQ, 1)
    bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tm_g,
                     const __grid_constant__ CUtensorMap tm_keys, BwdTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t g_full;      // G landed
  __shared__ __align__(8) uint64_t a_ready;     // the softmax warps wrote Q' into TMEM
  __shared__ __align__(8) uint64_t kv_full[kQStages];
  __shared__ __align__(8) uint64_t kv_empty[kQStages];
  __shared__ __align__(8) uint64_t sdp_full;    // S(j), dP(j) complete in TMEM
  __shared__ __align__(8) uint64_t sdp_free;    // the softmax warps loaded S(j), dP(j)
  __shared__ __align__(8) uint64_t ds_full;     // dS(j) written to TMEM
  __shared__ __align__(8) uint64_t ds_free;     // the products that read it completed
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sG = sbase, sK = sG + kTileGR;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int q0 = qt * kR;
  volatile int* abort_flag = &abort_sh;

  if (threadIdx.x == 0) {
    abort_sh = 0;
    mbar_init(smem_u32(&g_full), 1);
    mbar_init(smem_u32(&a_ready), kSoftmaxQ);
    for (int s = 0; s < kQStages; ++s) {
      mbar_init(smem_u32(&kv_full[s]), 1);
      mbar_init(smem_u32(&kv_empty[s]), 1);
    }
    mbar_init(smem_u32(&sdp_full), 1);
    mbar_init(smem_u32(&sdp_free), kSoftmaxQ);
    mbar_init(smem_u32(&ds_full), kSoftmaxQ);
    mbar_init(smem_u32(&ds_free), 1);
    fence_barrier_init();
  }
  if (warp == kMmaWarpQ) {
    tmem_alloc(smem_u32(&tmem_base_sh), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp == kProducerWarpQ) {
    // one copy per lane (lanes 0-3: the four 64-column blocks), so that a stage's copies go out
    // at once rather than one after another from a single thread; lane 0 waits and arms
    if (lane == 0) {
      const uint32_t gb = smem_u32(&g_full);
      mbar_arrive_expect_tx(gb, kTileGR);
      for (int i = 0; i < 3; ++i) tma_load_4d(sG + i * kBlkR, &tm_g, gb, 64 * i, h, q0, b);
    }
    bool ok = true;
    for (int j = 0; j < p.ns && ok; ++j) {
      const int s = j % kQStages;
      ok = __all_sync(0xffffffffu, lane != 0 || mbar_wait_or_abort(smem_u32(&kv_empty[s]),
                                                                   ((j / kQStages) & 1) ^ 1,
                                                                   abort_flag, p.dev_status));
      if (!ok) break;
      const uint32_t dst = sK + s * kTileS;
      const uint32_t fb = smem_u32(&kv_full[s]);
      if (lane == 0) mbar_arrive_expect_tx(fb, kTileS);
      __syncwarp();
      const int r0 = j < p.ns_ring ? j * kS : p.nc_pad + (j - p.ns_ring) * kS;
      if (lane < 4) tma_load_3d(dst + lane * kBlkS, &tm_keys, fb, 64 * lane, r0, b);
    }
  } else if (warp == kMmaWarpQ) {
    if (lane == 0) {
      // Order of issue: S/dP(j) once the softmax has loaded S/dP(j-1), then the dQ products of
      // sub-tile j-1 once its dS is in TMEM.
      bool ok = mbar_wait_or_abort(smem_u32(&a_ready), 0, abort_flag, p.dev_status) &&
                mbar_wait_or_abort(smem_u32(&g_full), 0, abort_flag, p.dev_status);
      for (int j = 0; j <= p.ns && ok; ++j) {
        if (j < p.ns) {
          const int s = j % kQStages;
          ok = mbar_wait_or_abort(smem_u32(&kv_full[s]), (j / kQStages) & 1, abort_flag,
                                  p.dev_status) &&
               (j == 0 || mbar_wait_or_abort(smem_u32(&sdp_free), (j - 1) & 1, abort_flag,
                                             p.dev_status));
          if (!ok) break;
          tc_fence_after();
          const uint32_t kt = sK + s * kTileS;
          mma_s_dp(tmem + kColS, tmem + kColDP, tmem + kColA, sG, kt);
          mma_commit(smem_u32(&sdp_full));
        }
        if (j >= 1) {
          const int jp = j - 1, sp = jp % kQStages;
          ok = mbar_wait_or_abort(smem_u32(&ds_full), jp & 1, abort_flag, p.dev_status);
          if (!ok) break;
          tc_fence_after();
          mma_tmem_by_sub224(tmem + kColAcc, tmem + kColDS, sK + sp * kTileS, jp > 0);
          mma_commit(smem_u32(&kv_empty[sp]));
          mma_commit(smem_u32(&ds_free));
        }
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
    row_to_tmem(tmem + lane_off + kColA,
                row_ok ? p.q + ((static_cast<int64_t>(b) * p.n_q + n) * p.H + h) * kD : nullptr,
                kAWords);
    tmem_wait_st();
    tc_fence_before();
    mbar_arrive(smem_u32(&a_ready));
    bool ok = true;
    for (int j = 0; j < p.ns && ok; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait_or_abort(smem_u32(&sdp_full), j & 1, abort_flag,
                                                      p.dev_status));
      if (!ok) break;
      tc_fence_after();
      const int valid = j < p.ns_ring ? min(kS, p.nc - j * kS)
                                      : min(kS, p.n_q - (j - p.ns_ring) * kS);
      uint32_t rs[64], rp[64];
      tmem_ld64_wait(tmem + lane_off + kColS, rs);
      tmem_ld64_wait(tmem + lane_off + kColDP, rp);
      tc_fence_before();
      mbar_arrive(smem_u32(&sdp_free));
      // pairs of columns on the packed fp32 pipe: x = S scale log2(e) - lse log2(e),
      // dS = exp2(x) (dP scale - Delta scale); columns past the valid keys get P = 0
      const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2), nl2 = f2_pack(-lse2, -lse2);
      const uint64_t dsc2 = f2_pack(p.scale, p.scale);
      const uint64_t nd2 = f2_pack(-delta * p.scale, -delta * p.scale);
      uint32_t w[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        float x0, x1;
        f2_unpack(f2_fma(f2_pack(__uint_as_float(rs[2 * i]), __uint_as_float(rs[2 * i + 1])), sc2,
                         nl2),
                  x0, x1);
        float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
        if (valid < kS) {
          p0 = 2 * i < valid ? p0 : 0.f;
          p1 = 2 * i + 1 < valid ? p1 : 0.f;
        }
        float d0, d1;
        f2_unpack(f2_mul(f2_fma(f2_pack(__uint_as_float(rp[2 * i]), __uint_as_float(rp[2 * i + 1])),
                                dsc2, nd2),
                         f2_pack(p0, p1)),
                  d0, d1);
        w[i] = pack_bf16x2(d0, d1);
      }
      // the dS columns were last read by the products of sub-tile j-1
      if (j >= 1)
        ok = __all_sync(0xffffffffu, mbar_wait_or_abort(smem_u32(&ds_free), (j - 1) & 1,
                                                        abort_flag, p.dev_status));
      if (!ok) break;
      {
        uint32_t w16[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) w16[i] = w[i];
        tmem_st16(tmem + lane_off + kColDS, w16);
#pragma unroll
        for (int i = 0; i < 16; ++i) w16[i] = w[16 + i];
        tmem_st16(tmem + lane_off + kColDS + 16, w16);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(smem_u32(&ds_full));
    }
    // the last dQ products completed: the (ns-1)-th completion of ds_free
    if (ok)
      ok = __all_sync(0xffffffffu, mbar_wait_or_abort(smem_u32(&ds_free), (p.ns - 1) & 1,
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
  if (warp == kMmaWarpQ) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------------------- key kernel

__global__ void __launch_bounds__(kThreadsK, 1)
    bwd_dkey_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_g, BwdTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t a_ready;              // the key tile is in TMEM
  __shared__ __align__(8) uint64_t qg_full[kKStages];   // Q'_i, G_i and their stats landed
  __shared__ __align__(8) uint64_t qg_empty[kKStages];  // the products of sub-tile i read them
  __shared__ __align__(8) uint64_t sdp_full;            // S^T, dP^T of sub-tile i complete
  __shared__ __align__(8) uint64_t sdp_free;            // the softmax warps loaded them
  __shared__ __align__(8) uint64_t pds_full;            // P^T, dS^T of sub-tile i in smem
  __shared__ __align__(8) uint64_t pds_free;            // the products that read them completed
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  // stage s (64 KB, Q' sub-tile stacked over G, see kBlkQG) at sStage + s * kKStage; then the P^T
  // and dS^T operands; then lse [64] and Delta [64] (512 B) of stage s at sStat + s * kStatBytes
  const uint32_t sStage = sbase;
  const uint32_t sP = sStage + kKStages * kKStage, sDS = sP + kOpBytes;
  const uint32_t sStat = sDS + kOpBytes;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int kt = blockIdx.x, grp = blockIdx.y, b = blockIdx.z;
  const int n_iter = p.heads_per_group * p.n_qs;
  volatile int* abort_flag = &abort_sh;

  if (threadIdx.x == 0) {
    abort_sh = 0;
    mbar_init(smem_u32(&a_ready), kSoftmaxK);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(smem_u32(&qg_full[s]), 1);
      mbar_init(smem_u32(&qg_empty[s]), 1);
    }
    mbar_init(smem_u32(&sdp_full), 1);
    mbar_init(smem_u32(&sdp_free), kSoftmaxK);
    mbar_init(smem_u32(&pds_full), kSoftmaxK);
    mbar_init(smem_u32(&pds_free), 1);
    fence_barrier_init();
  }
  // the G half of every stage's fourth block stays zero (no load writes it)
  for (int i = threadIdx.x; i < kKStages * kBlkS / 16; i += kThreadsK) {
    const int s = i / (kBlkS / 16), o = i % (kBlkS / 16);
    st_shared_v4(sStage + s * kKStage + 3 * kBlkQG + kBlkS + 16 * o, 0u, 0u, 0u, 0u);
  }
  fence_proxy_async_smem();
  if (warp == kMmaWarpK) {
    tmem_alloc(smem_u32(&tmem_base_sh), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp == kProducerWarpK) {
    // A stage's nine copies go out from nine lanes at once: issued one after another from a
    // single thread they take ~500 cycles, which adds to the load latency this kernel is
    // bound by.  Lane 0 waits for the stage and arms its barrier.
    bool ok = true;
    for (int it = 0; it < n_iter && ok; ++it) {
      const int s = it % kKStages;
      ok = __all_sync(0xffffffffu, lane != 0 || mbar_wait_or_abort(smem_u32(&qg_empty[s]),
                                                                   ((it / kKStages) & 1) ^ 1,
                                                                   abort_flag, p.dev_status));
      if (!ok) break;
      const int h = grp * p.heads_per_group + it / p.n_qs;
      const int q0 = (it % p.n_qs) * kS;
      // column statistics of the sub-tile: n_q is a multiple of 4, so both the source (row
      // (b, h) of [B, H, n_q] floats, column q0) and the size are 16-byte multiples
      const uint32_t stat_bytes = static_cast<uint32_t>(min(kS, p.n_q - q0)) * 4u;
      const int64_t so = (static_cast<int64_t>(b) * p.H + h) * p.n_q + q0;
      const uint32_t st = sStage + s * kKStage;
      const uint32_t fb = smem_u32(&qg_full[s]);
      if (lane == 0) mbar_arrive_expect_tx(fb, kTileS + kTileGS + 2 * stat_bytes);
      __syncwarp();
      // lanes 0-3: the four Q' boxes (the fourth covers columns 192-255: 224-255 lie past the
      // row and are filled with zeros, the padded rope block; the byte count is the full box);
      // lanes 4-6: the three G boxes; lanes 7, 8: lse and Delta
      if (lane < 4)
        tma_load_4d(st + lane * kBlkQG, &tm_q, fb, 64 * lane, h, q0, b);
      else if (lane < 7)
        tma_load_4d(st + (lane - 4) * kBlkQG + kBlkS, &tm_g, fb, 64 * (lane - 4), h, q0, b);
      else if (lane == 7)
        bulk_load(sStat + s * kStatBytes, p.lse + so, stat_bytes, fb);
      else if (lane == 8)
        bulk_load(sStat + s * kStatBytes + kS * 4, p.delta + so, stat_bytes, fb);
    }
  } else if (warp == kMmaWarpK) {
    if (lane == 0) {
      bool ok = mbar_wait_or_abort(smem_u32(&a_ready), 0, abort_flag, p.dev_status);
      for (int it = 0; it <= n_iter && ok; ++it) {
        if (it < n_iter) {
          const int s = it % kKStages;
          ok = mbar_wait_or_abort(smem_u32(&qg_full[s]), (it / kKStages) & 1, abort_flag,
                                  p.dev_status) &&
               (it == 0 || mbar_wait_or_abort(smem_u32(&sdp_free), (it - 1) & 1, abort_flag,
                                              p.dev_status));
          if (!ok) break;
          tc_fence_after();
          const uint32_t st = sStage + s * kKStage;
          mma_s_dp_stacked(tmem + kColS, tmem + kColA, st);
          mma_commit(smem_u32(&sdp_full));
        }
        if (it >= 1) {
          const int ip = it - 1, sp = ip % kKStages;
          ok = mbar_wait_or_abort(smem_u32(&pds_full), ip & 1, abort_flag, p.dev_status);
          if (!ok) break;
          tc_fence_after();
          const uint32_t stp = sStage + sp * kKStage;
          // key gradient dS^T Q' over all 256 columns first (it initialises the accumulator),
          // then the value gradient P^T G into the content columns
          mma_op_by_sub<256>(tmem + kColAcc, sDS, stp, kBlkQG, ip > 0);
          mma_op_by_sub<kDc>(tmem + kColAcc, sP, stp + kBlkS, kBlkQG, true);
          mma_commit(smem_u32(&qg_empty[sp]));
          mma_commit(smem_u32(&pds_free));
        }
      }
    }
  } else {
    // softmax warps: warps w and w + 4 share TMEM lanes 32 (w % 4) ...; each takes half of the
    // columns (ch = 0: sub-tile columns 0-31, 1: 32-63)
    const int quad = warp & 3, ch = warp >> 2;
    const int row = quad * 32 + lane;           // key row of the tile
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const bool key_ok = kt < p.nt_ring ? kt * kR + row < p.nc
                                       : (kt - p.nt_ring) * kR + row < p.n_q;
    const int prow = kt < p.nt_ring ? kt * kR + row : p.nc_pad + (kt - p.nt_ring) * kR + row;
    {
      // the key row into TMEM (bf16 pairs 0-63 by the first half, 64-111 by the second); rows
      // past the valid keys are zero in the padded copy
      const bf16* src = p.keys + (static_cast<int64_t>(b) * p.rows_ws + prow) * kBwdKeyWidth;
      row_to_tmem(tmem + lane_off + kColA + 64 * ch, src + 128 * ch, ch == 0 ? 64 : kAWords - 64);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(smem_u32(&a_ready));
    }
    bool ok = true;
    for (int it = 0; it < n_iter && ok; ++it) {
      const int s = it % kKStages;
      // S^T and dP^T of sub-tile it, and the column statistics the bulk copies of qg_full
      // brought (observed directly: the copies complete on that barrier)
      ok = __all_sync(0xffffffffu,
                      mbar_wait_or_abort(smem_u32(&sdp_full), it & 1, abort_flag,
                                         p.dev_status) &&
                          mbar_wait_or_abort(smem_u32(&qg_full[s]), (it / kKStages) & 1,
                                             abort_flag, p.dev_status));
      if (!ok) break;
      tc_fence_after();
      uint32_t rs[32], rp[32];
      tmem_ld32_wait(tmem + lane_off + kColS + 32 * ch, rs);
      tmem_ld32_wait(tmem + lane_off + kColDP + 32 * ch, rp);
      tc_fence_before();
      mbar_arrive(smem_u32(&sdp_free));
      // column statistics as packed pairs: -lse log2(e) and -Delta scale
      const float4* col_lse = reinterpret_cast<const float4*>(
          smem_raw + (sStat + s * kStatBytes - smem_u32(smem_raw))) + 8 * ch;
      const float4* col_delta = col_lse + kS / 4;
      const uint64_t nlog2e2 = f2_pack(-kLog2e, -kLog2e), nsc2 = f2_pack(-p.scale, -p.scale);
      uint64_t nl2[16], nd2[16];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 l = col_lse[i], d = col_delta[i];
        nl2[2 * i] = f2_mul(f2_pack(l.x, l.y), nlog2e2);
        nl2[2 * i + 1] = f2_mul(f2_pack(l.z, l.w), nlog2e2);
        nd2[2 * i] = f2_mul(f2_pack(d.x, d.y), nsc2);
        nd2[2 * i + 1] = f2_mul(f2_pack(d.z, d.w), nsc2);
      }
      // pairs of columns on the packed fp32 pipe; past the valid queries (or for a key row
      // past the valid keys) P and dS are 0, whatever the stale statistics there hold
      const int ncols = min(kS, p.n_q - (it % p.n_qs) * kS) - 32 * ch;
      const bool full = key_ok && ncols >= 32;
      const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2), dsc2 = f2_pack(p.scale, p.scale);
      uint32_t wp[16], wd[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float x0, x1, d0, d1;
        f2_unpack(f2_fma(f2_pack(__uint_as_float(rs[2 * i]), __uint_as_float(rs[2 * i + 1])), sc2,
                         nl2[i]),
                  x0, x1);
        float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
        f2_unpack(f2_mul(f2_fma(f2_pack(__uint_as_float(rp[2 * i]), __uint_as_float(rp[2 * i + 1])),
                                dsc2, nd2[i]),
                         f2_pack(p0, p1)),
                  d0, d1);
        if (!full) {
          const bool ok0 = key_ok && 2 * i < ncols, ok1 = key_ok && 2 * i + 1 < ncols;
          p0 = ok0 ? p0 : 0.f; d0 = ok0 ? d0 : 0.f;
          p1 = ok1 ? p1 : 0.f; d1 = ok1 ? d1 : 0.f;
        }
        wp[i] = pack_bf16x2(p0, p1);
        wd[i] = pack_bf16x2(d0, d1);
      }
      // the operands of sub-tile it-1 were read by its products
      if (it >= 1)
        ok = __all_sync(0xffffffffu, mbar_wait_or_abort(smem_u32(&pds_free), (it - 1) & 1,
                                                        abort_flag, p.dev_status));
      if (!ok) break;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        st_shared_v4(swz128(sP, row, 4 * ch + c), wp[4 * c], wp[4 * c + 1], wp[4 * c + 2], wp[4 * c + 3]);
        st_shared_v4(swz128(sDS, row, 4 * ch + c), wd[4 * c], wd[4 * c + 1], wd[4 * c + 2], wd[4 * c + 3]);
      }
      fence_proxy_async_smem();
      mbar_arrive(smem_u32(&pds_full));
    }
    if (ok)
      ok = __all_sync(0xffffffffu, mbar_wait_or_abort(smem_u32(&pds_free), (n_iter - 1) & 1,
                                                      abort_flag, p.dev_status));
    if (ok) {
      tc_fence_after();
      float* out = p.partial +
                   ((static_cast<int64_t>(grp) * gridDim.z + b) * p.rows_ws + prow) * kD;
      // columns [0, 128) by the first half, [128, 224) by the second
#pragma unroll 1
      for (int c = 128 * ch; c < (ch == 0 ? 128 : kD); c += 32) {
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
  if (warp == kMmaWarpK) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Writes the keys the tensor-core kernels read, row prow of sample b of the key workspace:
// [content latent (192) | rotated positional key (32) | 32 zeros]; rows past the valid ring
// keys (ring part [0, nc_pad)) or chunk keys (chunk part from nc_pad on) are zero.  One thread
// per 16-byte piece (8 bf16, 32 per row).
__global__ void bwd_pad_keys_kernel(const bf16* __restrict__ cache, const bf16* __restrict__ chunk_lat,
                                    const bf16* __restrict__ ws_rope, int B, int W, int tpf, int nc,
                                    int nc_pad, int n_q, int rows_ws, bf16* __restrict__ keys) {
  constexpr int kPieces = kBwdKeyWidth / 8;
  const int64_t total = static_cast<int64_t>(B) * rows_ws * kPieces;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int c8 = static_cast<int>(e % kPieces);
    const int64_t br = e / kPieces;
    const int prow = static_cast<int>(br % rows_ws), b = static_cast<int>(br / rows_ws);
    const bool ring = prow < nc_pad;
    const int m = ring ? prow : prow - nc_pad;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (ring ? m < nc : m < n_q) {
      if (c8 < kDc / 8) {
        const bf16* src = ring ? cache + (static_cast<int64_t>(b) * W * tpf + m) * kD
                               : chunk_lat + (static_cast<int64_t>(b) * n_q + m) * kD;
        v = *reinterpret_cast<const uint4*>(src + 8 * c8);
      } else if (c8 < kD / 8) {
        v = *reinterpret_cast<const uint4*>(ws_rope + br * kDr + 8 * (c8 - kDc / 8));
      }
    }
    *reinterpret_cast<uint4*>(keys + br * kBwdKeyWidth + 8 * c8) = v;
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
      const float2 v = *reinterpret_cast<const float2*>(
          partial + ((static_cast<int64_t>(gi) * B + b) * rows_ws + prow) * kD + 2 * pr);
      x0 += v.x;
      x1 += v.y;
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
  return d.dtype == MLA_BF16 && d.path != MLA_PATH_SIMT && d.d_c == kDc && d.d_rope == kDr &&
         d.n_q % 4 == 0;
}

namespace {

// Tensor maps of the backward's operands with row boxes of `rows` (128 for a tile a CTA owns, 64
// for a streamed sub-tile), all with 64-column boxes and the 128-byte swizzle; keys: the padded
// key copy.
struct BwdMaps {
  CUtensorMap q, g, keys;
};

mla_status make_bwd_maps(const Dims& d, const BwdArgs& a, const KeyWorkspace& kw,
                         const void* keys_tc, uint32_t rows, BwdMaps* m) {
  mla_status st;
  {
    const uint64_t dims[4] = {static_cast<uint64_t>(kD), static_cast<uint64_t>(d.H),
                              static_cast<uint64_t>(d.n_q), static_cast<uint64_t>(d.B)};
    const uint64_t strides[3] = {kD * 2ull, static_cast<uint64_t>(d.H) * kD * 2,
                                 static_cast<uint64_t>(d.n_q) * d.H * kD * 2};
    const uint32_t box[4] = {64, 1, rows, 1};
    if ((st = make_tmap_bf16(&m->q, a.q, 4, dims, strides, box, 128)) != MLA_OK) return st;
  }
  {
    const uint64_t dims[4] = {static_cast<uint64_t>(kDc), static_cast<uint64_t>(d.H),
                              static_cast<uint64_t>(d.n_q), static_cast<uint64_t>(d.B)};
    const uint64_t strides[3] = {kDc * 2ull, static_cast<uint64_t>(d.H) * kDc * 2,
                                 static_cast<uint64_t>(d.n_q) * d.H * kDc * 2};
    const uint32_t box[4] = {64, 1, rows, 1};
    if ((st = make_tmap_bf16(&m->g, a.d_o_lat, 4, dims, strides, box, 128)) != MLA_OK) return st;
  }
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(kBwdKeyWidth), static_cast<uint64_t>(kw.rows),
                              static_cast<uint64_t>(d.B)};
    const uint64_t strides[2] = {kBwdKeyWidth * 2ull,
                                 static_cast<uint64_t>(kw.rows) * kBwdKeyWidth * 2};
    const uint32_t box[3] = {64, rows, 1};
    if ((st = make_tmap_bf16(&m->keys, keys_tc, 3, dims, strides, box, 128)) != MLA_OK) return st;
  }
  return MLA_OK;
}

}  // namespace

mla_status attention_bwd_tc(const Dims& d, const BwdArgs& a, int n_valid, int first_frame,
                            const float* delta, const void* ws_rope, void* keys_tc,
                            float* partial, int groups, int32_t* dev_status, cudaStream_t s) {
  const KeyWorkspace kw = key_workspace_layout(d, n_valid);
  BwdMaps m128, m64;
  mla_status st = make_bwd_maps(d, a, kw, keys_tc, kR, &m128);
  if (st != MLA_OK) return st;
  if ((st = make_bwd_maps(d, a, kw, keys_tc, kS, &m64)) != MLA_OK) return st;
  BwdTcParams p;
  p.n_q = d.n_q; p.H = d.H; p.nc = kw.nc; p.nc_pad = kw.nc_pad;
  p.nt_ring = ceil_div(kw.nc, kR);
  p.nt = p.nt_ring + ceil_div(d.n_q, kR);
  p.ns_ring = ceil_div(kw.nc, kS);
  p.ns = p.ns_ring + ceil_div(d.n_q, kS);
  p.n_qs = ceil_div(d.n_q, kS);
  p.rows_ws = kw.rows; p.heads_per_group = d.H / groups;
  p.scale = d.scale; p.scale_log2 = d.scale * kLog2e;
  p.q = static_cast<const bf16*>(a.q); p.keys = static_cast<const bf16*>(keys_tc);
  p.lse = a.lse; p.delta = delta; p.d_q = a.d_q; p.partial = partial; p.dev_status = dev_status;
  {
    const int64_t pieces = static_cast<int64_t>(d.B) * kw.rows * (kBwdKeyWidth / 8);
    const int blocks = static_cast<int>(std::min<int64_t>((pieces + 255) / 256, 148 * 16));
    bwd_pad_keys_kernel<<<blocks, 256, 0, s>>>(
        static_cast<const bf16*>(a.cache), static_cast<const bf16*>(a.chunk_lat),
        static_cast<const bf16*>(ws_rope), d.B, d.W, d.tpf, kw.nc, kw.nc_pad, d.n_q, kw.rows,
        static_cast<bf16*>(keys_tc));
    MLA_LAUNCH_CHECK("bwd_pad_keys");
  }
  MLA_CUDA_TRY(cudaFuncSetAttribute(bwd_dq_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    kSmemQ));
  MLA_CUDA_TRY(cudaFuncSetAttribute(bwd_dkey_tc_kernel,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemK));
  // dQ kernel: owns a 128-row query tile (Q' copied into TMEM by its threads, G by 128-row
  // boxes), streams 64-key sub-tiles
  dim3 gq(ceil_div(d.n_q, kR), d.H, d.B);
  bwd_dq_tc_kernel<<<gq, kThreadsQ, kSmemQ, s>>>(m128.g, m64.keys, p);
  MLA_LAUNCH_CHECK("bwd_dq_tc");
  // key kernel: owns a 128-key tile (copied into TMEM by its threads), streams 64-query
  // sub-tiles (Q', G by 64-row boxes)
  dim3 gk(p.nt, groups, d.B);
  bwd_dkey_tc_kernel<<<gk, kThreadsK, kSmemK, s>>>(m64.q, m64.g, p);
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
