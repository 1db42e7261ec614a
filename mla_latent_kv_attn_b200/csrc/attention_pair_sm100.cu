// attention_pair_sm100.cu - the latent-space attention of attention_sm100.cu, run by CTA pairs
// whose tensor cores execute every MMA together (tcgen05 cta_group::2).
//
// VideoMLA (hyper.ai summary, "Method"): every head scores q_nope.k_nope + q_rope.k_rope against
// keys rebuilt from the one cached latent; in absorbed form all heads share the same keys
// K'_m = [c_m || RoPE(k_R,m)] and values c_m (MQA).  That sharing is what a pair exploits: a
// cluster of two CTAs takes two heads of the same 128-row query tile of one sample, and each
// pair MMA multiplies the two heads' 256 query rows by one key tile whose rows are split
// between the two CTAs' shared memory.
//
//   S_j  = Q K'_j^T     M=256 (128 rows per CTA: its own head), N=128 keys: the even CTA holds
//                       keys 0..63 of the tile, the odd one keys 64..127 (K-major, 128B swizzle)
//   O   += P_j V_j      M=256, N=DC: the even CTA holds value columns 0..DC/2-1 of all 128 keys,
//                       the odd one columns DC/2.. (MN-major, 64B swizzle); P from each CTA's TMEM
//   o    = O_lat [W_UV,h ; W_UV,h+1]^T   (epilogue) M=256, N=256: each CTA holds its head's
//                       W_UV tile and keeps the 128 output columns of its own head
//
// Per CTA and key tile that is 28 KB of keys and 24 KB of values (52 KB) instead of one 56 KB
// tile read twice by the tensor core, so the query tile stays in shared memory and TMEM has
// room for two S buffers: S0 [0,128), S1 [128,256), O [256,256+DC), P [256+DC, +64).  With two S
// buffers QK(j+1) never waits for the softmax to have loaded S(j); the softmax of tile j and the
// products of neighbouring tiles overlap.
//
// The key halves and the value halves travel in two rings of their own: a key stage is refilled
// as soon as QK of its tile has completed, a full PV earlier than a shared stage would be, so
// the load latency of the next key tiles stays off the critical path with three stages each.
//
// Roles (256 threads per CTA, the same in both CTAs except that only the even CTA issues MMAs):
//   warps 0-3  softmax of the CTA's own 128 rows (one TMEM lane each): as in attention_sm100.cu
//   warp 4     TMA producer of the query tile and key halves (then the W_UV tile); completion is
//              counted on the even CTA's barriers
//   warp 5     TMEM allocation (both CTAs, collectively); in the even CTA one thread issues QK
//   warp 6     in the even CTA one thread issues PV and the W_UV epilogue
//   warp 7     TMA producer of the value halves
// Barriers that a thread of either CTA arrives on live in the even CTA (counts: one TMA arrival,
// or one arrival per softmax warp of both CTAs); barriers the tensor cores signal exist in both
// CTAs and receive the pair MMAs' commits by cluster multicast.  Every wait is bounded.
#include "exp2.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace mla {

namespace {

using namespace sm100;

constexpr int kBM = 128;           // query rows per CTA
constexpr int kBN = kKeyTile;      // keys per tile (both CTAs)
constexpr int kHalfN = kBN / 2;    // keys per CTA in the QK operand
constexpr int kDh = 128;           // head width of the W_UV epilogue
constexpr int kSoftmaxWarps = 4;
constexpr int kProducerWarp = 4;   // query tile, key halves (and the W_UV tile)
constexpr int kQkWarp = 5;
constexpr int kPvWarp = 6;
constexpr int kVProducerWarp = 7;  // value halves
constexpr int kThreads = 256;
constexpr int kSmemMax = 227 * 1024;
constexpr uint32_t kTmemCols = 512;
constexpr uint16_t kBothCtas = 0x3;
constexpr int kPolyPairsPer8Pair = 2;   // share of FMA-pipe exponentials (pairs out of every 8)

template <int DC_, int DR_>
struct PairShape {
  static constexpr int DC = DC_, DR = DR_, D = DC + DR;
  static_assert(DC == 128 || DC == 192, "pair kernel: DC 128 or 192 (TMEM: 2 S + O + P)");
  static_assert(DR == 16 || DR == 32 || DR == 64, "DR must be 16, 32 or 64");
  static constexpr int kCBlk = DC / 64;                     // 64-column content blocks
  static constexpr int kRopeBytes = DR * 2;
  static constexpr uint32_t kRopeSwz = DR == 16 ? kSwizzle32B : DR == 32 ? kSwizzle64B
                                                                         : kSwizzle128B;
  static constexpr int kRopeSbo = 8 * kRopeBytes;
  static constexpr int kRopeKSteps = DR / 16;
  // query tile: kCBlk blocks of 128 rows x 128 B (128B swizzle), then 128 rows of DR values
  static constexpr int kQBlk = kBM * 128;
  static constexpr int kQTile = kCBlk * kQBlk + kBM * kRopeBytes;
  // Two rings of the same depth, filled and freed independently:
  //   key stage:   the CTA's 64 keys for QK (kCBlk blocks of 64 rows x 128 B, then 64 rope
  //                rows); free once QK of its tile has completed
  //   value stage: the CTA's DC/2 value columns of all 128 keys (DC/64 blocks of 128 rows x
  //                64 B, 64B swizzle); free once PV of its tile has completed
  static constexpr int kOwnBlk = kHalfN * 128;
  static constexpr int kOwn = kCBlk * kOwnBlk + kHalfN * kRopeBytes;
  static constexpr int kVBlk = kBN * 64;
  static constexpr int kVCols = DC / 2;
  static constexpr int kVBlocks = kVCols / 32;
  static constexpr int kVStage = kVBlocks * kVBlk;
  static constexpr int kFit = (kSmemMax - 1024 - kQTile) / (kOwn + kVStage);
  static constexpr int kStages = kFit < 4 ? kFit : 4;
  static_assert(kStages >= 2, "too few stages fit in shared memory");
  static_assert(kOwn % 1024 == 0 && kVStage % 1024 == 0, "stage regions must stay 1 KB aligned");
  static constexpr int kSmem = kQTile + kStages * (kOwn + kVStage) + 1024;
  static constexpr int kWTile = kCBlk * kQBlk;              // W_UV_h: 128 rows x DC
  static_assert(kWTile <= kStages * kOwn, "the W_UV tile goes into the key ring");
  static constexpr uint32_t kColO = 256;
  static constexpr uint32_t kColP = kColO + DC;
  static_assert(kColP + kBN / 2 <= kTmemCols, "TMEM: S0, S1, O and P must fit");
};

struct PairParams {
  int n_q, H, nc, nc_pad, nt_ring, nt;
  float scale_log2;
  int has_w_uv;
  void* out;
  float* lse;
  int32_t* dev_status;
};

// p = 2^(s * scale_log2 - m) for one row of a key tile (as in attention_sm100.cu).
template <bool kPoly>
__device__ __forceinline__ float pair_exp_row(const float (&s)[kBN], float scale_log2, float m,
                                              uint32_t (&w)[kBN / 2]) {
  const uint64_t sc2 = f2_pack(scale_log2, scale_log2);
  const uint64_t nm2 = f2_pack(-m, -m);
  uint64_t sum2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
  for (int i = 0; i < kBN / 2; ++i) {
    float x0, x1, p0, p1;
    f2_unpack(f2_fma(f2_pack(s[2 * i], s[2 * i + 1]), sc2, nm2), x0, x1);
    if (kPoly && (i & 7) < kPolyPairsPer8Pair) {
      exp2_poly_pair(x0, x1, p0, p1);
    } else {
      p0 = fast_exp2(x0);
      p1 = fast_exp2(x1);
    }
    sum2[i & 3] = f2_add(sum2[i & 3], f2_pack(p0, p1));
    w[i] = pack_bf16x2(p0, p1);
  }
  const uint64_t t2 = f2_add(f2_add(sum2[0], sum2[1]), f2_add(sum2[2], sum2[3]));
  float l0, l1;
  f2_unpack(t2, l0, l1);
  return l0 + l1;
}

// Waits use the default acquire (CTA scope) whoever arrives: the data behind every per-tile
// barrier is TMEM or TMA-written shared memory, ordered by tcgen05 fences and the async proxy;
// the one hand-off of generic shared-memory writes (O_lat) is released at cluster scope.
__device__ __forceinline__ bool pwait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                      int32_t* dev_status) {
  return mbar_wait_or_abort(bar, parity, abort_flag, dev_status);
}

template <int DC, int DR>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    attention_pair_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_qr,
                          const __grid_constant__ CUtensorMap tm_cache_k,
                          const __grid_constant__ CUtensorMap tm_cache_v,
                          const __grid_constant__ CUtensorMap tm_chunk_k,
                          const __grid_constant__ CUtensorMap tm_chunk_v,
                          const __grid_constant__ CUtensorMap tm_ws,
                          const __grid_constant__ CUtensorMap tm_wuv, PairParams p) {
  using Sh = PairShape<DC, DR>;
  constexpr int kCBlk = Sh::kCBlk;
  constexpr int kStages = Sh::kStages;
  constexpr uint32_t kColO = Sh::kColO, kColP = Sh::kColP;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t q_full;            // even CTA: both query tiles landed
  __shared__ __align__(8) uint64_t k_full[kStages];   // even CTA: both CTAs' key halves landed
  __shared__ __align__(8) uint64_t k_empty[kStages];  // both: QK of the stage's tile done
  __shared__ __align__(8) uint64_t v_full[kStages];   // even CTA: both CTAs' value halves landed
  __shared__ __align__(8) uint64_t v_empty[kStages];  // both: PV of the stage's tile done
  __shared__ __align__(8) uint64_t s_full[2];         // both: S buffer written
  __shared__ __align__(8) uint64_t s_free[2];         // even CTA: 8 softmax warps loaded it
  __shared__ __align__(8) uint64_t p_full;            // even CTA: 8 softmax warps wrote P
  __shared__ __align__(8) uint64_t pv_done;           // both: PV(j) done (O and P free)
  __shared__ __align__(8) uint64_t w_full;            // even CTA: both W_UV tiles landed
  __shared__ __align__(8) uint64_t olat_full;         // even CTA: 8 softmax warps wrote O_lat
  __shared__ __align__(8) uint64_t epi_done;          // both: epilogue product done
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sQ = sbase;
  const uint32_t sK0 = sbase + Sh::kQTile;                       // key ring
  const uint32_t sV0 = sK0 + kStages * Sh::kOwn;                  // value ring
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int h = blockIdx.x, qt = blockIdx.y, b = blockIdx.z;
  const int q0 = qt * kBM;
  volatile int* abort_flag = &abort_sh;

  if (threadIdx.x == 0) {
    abort_sh = 0;
    mbar_init(smem_u32(&q_full), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&k_full[s]), 1);
      mbar_init(smem_u32(&k_empty[s]), 1);
      mbar_init(smem_u32(&v_full[s]), 1);
      mbar_init(smem_u32(&v_empty[s]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&s_full[i]), 1);
      mbar_init(smem_u32(&s_free[i]), 2 * kSoftmaxWarps);
    }
    mbar_init(smem_u32(&p_full), 2 * kSoftmaxWarps);
    mbar_init(smem_u32(&pv_done), 1);
    mbar_init(smem_u32(&w_full), 1);
    mbar_init(smem_u32(&olat_full), 2 * kSoftmaxWarps);
    mbar_init(smem_u32(&epi_done), 1);
    fence_barrier_init();
  }
  if (warp == kQkWarp) {
    tmem_alloc_pair(smem_u32(&tmem_base_sh), kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  // both CTAs' barriers are initialised (and TMEM allocated) before either CTA signals the other
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------------ TMA producer: Q, keys
    if (lane == 0) {
      tma_prefetch_desc(&tm_chunk_k);
      tma_prefetch_desc(&tm_ws);
      tma_prefetch_desc(&tm_q);
      // completions are counted on the even CTA's barriers
      const uint32_t qb = map_to_cta(smem_u32(&q_full), 0);
      if (leader) mbar_arrive_expect_tx(smem_u32(&q_full), 2 * Sh::kQTile);
      for (int i = 0; i < kCBlk; ++i)
        tma_load_4d_pair(sQ + i * Sh::kQBlk, &tm_q, qb, 64 * i, h, q0, b);
      tma_load_4d_pair(sQ + kCBlk * Sh::kQBlk, &tm_qr, qb, DC, h, q0, b);
      bool ok = true;
      for (int j = 0; j < p.nt && ok; ++j) {
        const int s = j % kStages;
        ok = pwait(smem_u32(&k_empty[s]), ((j / kStages) & 1) ^ 1, abort_flag, p.dev_status);
        if (!ok) break;
        const uint32_t own = sK0 + s * Sh::kOwn;
        const uint32_t fb = map_to_cta(smem_u32(&k_full[s]), 0);
        if (leader) mbar_arrive_expect_tx(smem_u32(&k_full[s]), 2 * Sh::kOwn);
        const bool ring = j < p.nt_ring;
        const int r0 = ring ? j * kBN : (j - p.nt_ring) * kBN;       // tile's first key row
        const int rk = r0 + kHalfN * static_cast<int>(rank);          // this CTA's QK keys
        const CUtensorMap* mk = ring ? &tm_cache_k : &tm_chunk_k;
        for (int i = 0; i < kCBlk; ++i) tma_load_3d_pair(own + i * Sh::kOwnBlk, mk, fb, 64 * i, rk, b);
        tma_load_3d_pair(own + kCBlk * Sh::kOwnBlk, &tm_ws, fb, 0, ring ? rk : p.nc_pad + rk, b);
      }
      if (ok && p.has_w_uv) {
        // W_UV of this CTA's head into the key ring once every key stage is free
        for (int jj = p.nt; jj < p.nt + kStages && ok; ++jj)
          ok = pwait(smem_u32(&k_empty[jj % kStages]), ((jj / kStages) & 1) ^ 1, abort_flag,
                     p.dev_status);
        if (ok) {
          const uint32_t wb = map_to_cta(smem_u32(&w_full), 0);
          if (leader) mbar_arrive_expect_tx(smem_u32(&w_full), 2 * Sh::kWTile);
          for (int i = 0; i < kCBlk; ++i)
            tma_load_2d_pair(sK0 + i * Sh::kQBlk, &tm_wuv, wb, 64 * i, h * kDh);
        }
      }
    }
  } else if (warp == kVProducerWarp) {
    // ------------------------------------------------------------------ TMA producer: values
    if (lane == 0) {
      tma_prefetch_desc(&tm_chunk_v);
      bool ok = true;
      for (int j = 0; j < p.nt && ok; ++j) {
        const int s = j % kStages;
        ok = pwait(smem_u32(&v_empty[s]), ((j / kStages) & 1) ^ 1, abort_flag, p.dev_status);
        if (!ok) break;
        const uint32_t vreg = sV0 + s * Sh::kVStage;
        const uint32_t fb = map_to_cta(smem_u32(&v_full[s]), 0);
        if (leader) mbar_arrive_expect_tx(smem_u32(&v_full[s]), 2 * Sh::kVStage);
        const bool ring = j < p.nt_ring;
        const int r0 = ring ? j * kBN : (j - p.nt_ring) * kBN;
        const CUtensorMap* mv = ring ? &tm_cache_v : &tm_chunk_v;
        for (int i = 0; i < Sh::kVBlocks; ++i)
          tma_load_3d_pair(vreg + i * Sh::kVBlk, mv, fb, Sh::kVCols * static_cast<int>(rank) + 32 * i,
                           r0, b);
      }
    }
  } else if (warp == kQkWarp || warp == kPvWarp) {
    // ------------------------------------------------------------------ pair MMA issuers
    if (leader && lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(2 * kBM, kBN, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(2 * kBM, DC, 0, 1);
      constexpr uint32_t idesc_uv = idesc_bf16_f32(2 * kBM, 2 * kDh, 0, 0);
      // descriptors are built once; an operand at byte offset `off` is the descriptor + off/16
      const uint64_t q_c = smem_desc(sQ, 16, 1024, kSwizzle128B);
      const uint64_t q_r = smem_desc(sQ + kCBlk * Sh::kQBlk, 16, Sh::kRopeSbo, Sh::kRopeSwz);
      const uint64_t k_c0 = smem_desc(sK0, 16, 1024, kSwizzle128B);
      const uint64_t k_r0 = smem_desc(sK0 + kCBlk * Sh::kOwnBlk, 16, Sh::kRopeSbo, Sh::kRopeSwz);
      const uint64_t v_0 = smem_desc(sV0, Sh::kVBlk, 512, kSwizzle64B);
      constexpr uint32_t kOwnD = Sh::kOwn >> 4, kVStageD = Sh::kVStage >> 4;
      bool ok = true;
      if (warp == kQkWarp) {
        ok = pwait(smem_u32(&q_full), 0, abort_flag, p.dev_status);
        for (int j = 0; j < p.nt && ok; ++j) {
          const int s = j % kStages;
          ok = pwait(smem_u32(&k_full[s]), (j / kStages) & 1, abort_flag, p.dev_status);
          // S buffer j&1 was loaded by both CTAs' softmax warps (tile j-2)
          if (ok && j >= 2)
            ok = pwait(smem_u32(&s_free[j & 1]), ((j - 2) >> 1) & 1, abort_flag, p.dev_status);
          if (!ok) break;
          tc_fence_after();
          const uint32_t d = tmem + (j & 1) * kBN;
          const uint64_t kc = k_c0 + static_cast<uint32_t>(s) * kOwnD;
          const uint64_t kr = k_r0 + static_cast<uint32_t>(s) * kOwnD;
#pragma unroll
          for (int blk = 0; blk < kCBlk; ++blk)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ss_pair(d, q_c + (blk * (Sh::kQBlk >> 4) + 2 * kk),
                          kc + (blk * (Sh::kOwnBlk >> 4) + 2 * kk), idesc_qk,
                          (blk | kk) != 0 ? 1u : 0u);
#pragma unroll
          for (int kk = 0; kk < Sh::kRopeKSteps; ++kk)
            mma_ss_pair(d, q_r + 2 * kk, kr + 2 * kk, idesc_qk, 1u);
          mma_commit_pair(smem_u32(&s_full[j & 1]), kBothCtas);
          mma_commit_pair(smem_u32(&k_empty[s]), kBothCtas);
        }
      } else {
        for (int j = 0; j < p.nt && ok; ++j) {
          const int s = j % kStages;
          ok = pwait(smem_u32(&v_full[s]), (j / kStages) & 1, abort_flag, p.dev_status) &&
               pwait(smem_u32(&p_full), j & 1, abort_flag, p.dev_status);
          if (!ok) break;
          tc_fence_after();
          const uint64_t vd = v_0 + static_cast<uint32_t>(s) * kVStageD;
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk)
            // keys kk*16 .. +15: 16 rows of 64 B further per step (1024 B = 64 units)
            mma_ts_pair(tmem + kColO, tmem + kColP + kk * 8, vd + 64 * kk, idesc_pv,
                        (j | kk) != 0 ? 1u : 0u);
          mma_commit_pair(smem_u32(&v_empty[s]), kBothCtas);
          mma_commit_pair(smem_u32(&pv_done), kBothCtas);
        }
        if (ok && p.has_w_uv) {
          ok = pwait(smem_u32(&w_full), 0, abort_flag, p.dev_status) &&
               mbar_wait_cluster_or_abort(smem_u32(&olat_full), 0, abort_flag, p.dev_status);
          if (ok) {
            tc_fence_after();
            const uint64_t o_c = smem_desc(sQ, 16, 1024, kSwizzle128B);     // O_lat over Q
            const uint64_t w_c = smem_desc(sK0, 16, 1024, kSwizzle128B);    // W_UV: key ring
#pragma unroll
            for (int blk = 0; blk < kCBlk; ++blk)
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_ss_pair(tmem, o_c + (blk * (Sh::kQBlk >> 4) + 2 * kk),
                            w_c + (blk * (Sh::kQBlk >> 4) + 2 * kk), idesc_uv,
                            (blk | kk) != 0 ? 1u : 0u);
            mma_commit_pair(smem_u32(&epi_done), kBothCtas);
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax warps 0..3
    const int row = warp * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const int n = q0 + row;
    const uint32_t s_free_l0 = map_to_cta(smem_u32(&s_free[0]), 0);
    const uint32_t s_free_l1 = map_to_cta(smem_u32(&s_free[1]), 0);
    const uint32_t p_full_l = map_to_cta(smem_u32(&p_full), 0);
    const uint32_t olat_full_l = map_to_cta(smem_u32(&olat_full), 0);
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < p.nt; ++j) {
      const int sb = j & 1;
      ok = __all_sync(0xffffffffu,
                      pwait(smem_u32(&s_full[sb]), (j >> 1) & 1, abort_flag, p.dev_status));
      if (!ok) break;
      tc_fence_after();
      float s[kBN];
      {
        uint32_t r[kBN];
        tmem_ld128_wait(tmem + lane_off + sb * kBN, r);
#pragma unroll
        for (int i = 0; i < kBN; ++i) s[i] = __uint_as_float(r[i]);
      }
      // S(j) is in registers: one arrival per warp frees its buffer for QK(j+2)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(sb ? s_free_l1 : s_free_l0);
      const int valid = j < p.nt_ring ? min(kBN, p.nc - j * kBN)
                                      : min(kBN, p.n_q - (j - p.nt_ring) * kBN);
      if (valid < kBN) {
#pragma unroll
        for (int c = 0; c < kBN; ++c)
          if (c >= valid) s[c] = -INFINITY;
      }
      float mx;
      {
        float m8[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          float a = fmax3(s[u], s[u + 8], s[u + 16]);
#pragma unroll
          for (int c = 24; c < kBN - 8; c += 16) a = fmax3(a, s[c + u], s[c + 8 + u]);
          m8[u] = fmaxf(a, s[kBN - 8 + u]);
        }
        mx = fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7])) *
             p.scale_log2;
      }
      bool rescale = false;
      float alpha = 1.f;
      if (j == 0) {
        m_run = mx;
      } else if (__any_sync(0xffffffffu, mx > m_run + 8.f)) {
        const float m_new = fmaxf(m_run, mx);
        alpha = fast_exp2(m_run - m_new);
        l_run *= alpha;
        m_run = m_new;
        rescale = true;
      }
      uint32_t w[kBN / 2];
      if (valid == kBN) l_run += pair_exp_row<true>(s, p.scale_log2, m_run, w);
      else l_run += pair_exp_row<false>(s, p.scale_log2, m_run, w);
      // P and O are free once PV(j-1) has completed
      if (j > 0) {
        ok = __all_sync(0xffffffffu, pwait(smem_u32(&pv_done), (j - 1) & 1, abort_flag, p.dev_status));
        if (!ok) break;
        tc_fence_after();
      }
      if (rescale) {
#pragma unroll 1
        for (int c = 0; c < DC; c += 16) {
          uint32_t r[16];
          tmem_ld16_wait(tmem + lane_off + kColO + c, r);
#pragma unroll
          for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
          tmem_st16(tmem + lane_off + kColO + c, r);
        }
      }
#pragma unroll
      for (int c = 0; c < kBN / 2; c += 16) {
        uint32_t w16[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) w16[i] = w[c + i];
        tmem_st16(tmem + lane_off + kColP + c, w16);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(p_full_l);
    }
    if (ok)
      ok = __all_sync(0xffffffffu, pwait(smem_u32(&pv_done), (p.nt - 1) & 1, abort_flag, p.dev_status));
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.f / l_run;
      if (p.lse != nullptr && n < p.n_q)
        p.lse[(static_cast<int64_t>(b) * p.H + h) * p.n_q + n] =
            (m_run + log2f(l_run)) * 0.69314718055994530942f;
      if (!p.has_w_uv) {
        bf16* orow = static_cast<bf16*>(p.out) + ((static_cast<int64_t>(b) * p.n_q + n) * p.H + h) * DC;
#pragma unroll 1
        for (int c = 0; c < DC; c += 32) {
          uint32_t r[32];
          tmem_ld32_wait(tmem + lane_off + kColO + c, r);
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            w[i] = pack_bf16x2(__uint_as_float(r[2 * i]) * inv_l, __uint_as_float(r[2 * i + 1]) * inv_l);
          if (n < p.n_q) {
            uint4* d4 = reinterpret_cast<uint4*>(orow + c);
#pragma unroll
            for (int i = 0; i < 4; ++i) d4[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
          }
        }
      } else {
        // O_lat (bf16) over the dead query tile, 128B-swizzled K-major: the A operand of the
        // epilogue product (every QK has completed: the softmax waited for the last S)
        uint8_t* qsm = smem_raw + (sQ - smem_u32(smem_raw));
#pragma unroll 1
        for (int c = 0; c < DC; c += 32) {
          uint32_t r[32];
          tmem_ld32_wait(tmem + lane_off + kColO + c, r);
          const int blk = c / 64;
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            const int chunk = (c % 64) / 8 + ch;
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(r[8 * ch + 0]) * inv_l, __uint_as_float(r[8 * ch + 1]) * inv_l);
            v.y = pack_bf16x2(__uint_as_float(r[8 * ch + 2]) * inv_l, __uint_as_float(r[8 * ch + 3]) * inv_l);
            v.z = pack_bf16x2(__uint_as_float(r[8 * ch + 4]) * inv_l, __uint_as_float(r[8 * ch + 5]) * inv_l);
            v.w = pack_bf16x2(__uint_as_float(r[8 * ch + 6]) * inv_l, __uint_as_float(r[8 * ch + 7]) * inv_l);
            const int off = blk * Sh::kQBlk + row * 128 + ((chunk ^ (row & 7)) * 16);
            *reinterpret_cast<uint4*>(qsm + off) = v;
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(olat_full_l);
        ok = __all_sync(0xffffffffu, pwait(smem_u32(&epi_done), 0, abort_flag, p.dev_status));
        if (ok) {
          tc_fence_after();
          // this CTA's head is the N half `rank` of the pair product
          const uint32_t col0 = rank * kDh;
          bf16* orow = static_cast<bf16*>(p.out) +
                       (static_cast<int64_t>(b) * p.n_q + n) * (static_cast<int64_t>(p.H) * kDh) +
                       static_cast<int64_t>(h) * kDh;
#pragma unroll 1
          for (int c = 0; c < kDh; c += 32) {
            uint32_t r[32];
            tmem_ld32_wait(tmem + lane_off + col0 + c, r);
            uint32_t w[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              w[i] = pack_bf16x2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
            if (n < p.n_q) {
              uint4* d4 = reinterpret_cast<uint4*>(orow + c);
#pragma unroll
              for (int i = 0; i < 4; ++i) d4[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  // neither CTA leaves (or frees TMEM) while the other may still use its shared memory
  cluster_sync_all();
  if (warp == kQkWarp) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

template <int DC, int DR>
mla_status attention_pair_impl(const Dims& d, const AttnArgs& a, int n_valid, cudaStream_t s) {
  using Sh = PairShape<DC, DR>;
  constexpr int kD = Sh::D;
  const KeyWorkspace kw = key_workspace_layout(d, n_valid);
  CUtensorMap tq, tqr, tck, tcv, thk, thv, tws, twuv;
  mla_status st;
  {
    const uint64_t dims[4] = {static_cast<uint64_t>(kD), static_cast<uint64_t>(d.H),
                              static_cast<uint64_t>(d.n_q), static_cast<uint64_t>(d.B)};
    const uint64_t strides[3] = {kD * 2ull, static_cast<uint64_t>(d.H) * kD * 2,
                                 static_cast<uint64_t>(d.n_q) * d.H * kD * 2};
    const uint32_t box[4] = {64, 1, kBM, 1};
    if ((st = make_tmap_bf16(&tq, a.q, 4, dims, strides, box, 128)) != MLA_OK) return st;
    const uint32_t box_r[4] = {DR, 1, kBM, 1};
    if ((st = make_tmap_bf16(&tqr, a.q, 4, dims, strides, box_r, Sh::kRopeBytes)) != MLA_OK)
      return st;
  }
  // content of keys: QK halves (64 columns x 64 keys, 128B swizzle) and value columns (32 x 128
  // keys, 64B swizzle), over the chunk latents and the valid ring rows
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(kD), static_cast<uint64_t>(d.n_q),
                              static_cast<uint64_t>(d.B)};
    const uint64_t strides[2] = {kD * 2ull, static_cast<uint64_t>(d.n_q) * kD * 2};
    const uint32_t box_k[3] = {64, kHalfN, 1};
    const uint32_t box_v[3] = {32, kBN, 1};
    if ((st = make_tmap_bf16(&thk, a.chunk_lat, 3, dims, strides, box_k, 128)) != MLA_OK) return st;
    if ((st = make_tmap_bf16(&thv, a.chunk_lat, 3, dims, strides, box_v, 64)) != MLA_OK) return st;
  }
  if (kw.nc > 0) {
    const uint64_t dims[3] = {static_cast<uint64_t>(kD), static_cast<uint64_t>(kw.nc),
                              static_cast<uint64_t>(d.B)};
    const uint64_t strides[2] = {kD * 2ull, static_cast<uint64_t>(d.W) * d.tpf * kD * 2};
    const uint32_t box_k[3] = {64, kHalfN, 1};
    const uint32_t box_v[3] = {32, kBN, 1};
    if ((st = make_tmap_bf16(&tck, a.cache, 3, dims, strides, box_k, 128)) != MLA_OK) return st;
    if ((st = make_tmap_bf16(&tcv, a.cache, 3, dims, strides, box_v, 64)) != MLA_OK) return st;
  } else {
    tck = thk;   // never read: no ring tiles
    tcv = thv;
  }
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(DR), static_cast<uint64_t>(kw.rows),
                              static_cast<uint64_t>(d.B)};
    const uint64_t strides[2] = {DR * 2ull, static_cast<uint64_t>(kw.rows) * DR * 2};
    const uint32_t box[3] = {DR, kHalfN, 1};
    if ((st = make_tmap_bf16(&tws, a.ws, 3, dims, strides, box, Sh::kRopeBytes)) != MLA_OK)
      return st;
  }
  if (a.w_uv != nullptr) {
    const uint64_t dims[2] = {static_cast<uint64_t>(DC), static_cast<uint64_t>(d.H) * kDh};
    const uint64_t strides[1] = {DC * 2ull};
    const uint32_t box[2] = {64, kDh};
    if ((st = make_tmap_bf16(&twuv, a.w_uv, 2, dims, strides, box, 128)) != MLA_OK) return st;
  } else {
    twuv = thk;   // never read
  }
  PairParams p;
  p.n_q = d.n_q; p.H = d.H; p.nc = kw.nc; p.nc_pad = kw.nc_pad;
  p.nt_ring = ceil_div(kw.nc, kBN);
  p.nt = p.nt_ring + ceil_div(d.n_q, kBN);
  p.scale_log2 = d.scale * 1.4426950408889634f;
  p.has_w_uv = a.w_uv != nullptr;
  p.out = a.out; p.lse = a.lse; p.dev_status = a.dev_status;
  MLA_CUDA_TRY(cudaFuncSetAttribute(attention_pair_kernel<DC, DR>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, Sh::kSmem));
  dim3 grid(d.H, ceil_div(d.n_q, kBM), d.B);     // clusters: heads (2c, 2c+1)
  attention_pair_kernel<DC, DR><<<grid, kThreads, Sh::kSmem, s>>>(tq, tqr, tck, tcv, thk, thv, tws,
                                                                  twuv, p);
  MLA_LAUNCH_CHECK("attention_pair");
  return MLA_OK;
}

}  // namespace

bool tc_attention_pair_supported(const Dims& d, bool has_w_uv) {
  return d.dtype == MLA_BF16 && (d.d_c == 128 || d.d_c == 192) &&
         (d.d_rope == 16 || d.d_rope == 32 || d.d_rope == 64) && d.H % 2 == 0 &&
         (!has_w_uv || d.d_head == kDh);
}

mla_status attention_tc_pair(const Dims& d, const AttnArgs& a, int n_valid, cudaStream_t s) {
#define MLA_PAIR_CASE(DC, DR) \
  if (d.d_c == DC && d.d_rope == DR) return attention_pair_impl<DC, DR>(d, a, n_valid, s);
  MLA_PAIR_CASE(128, 16) MLA_PAIR_CASE(128, 32) MLA_PAIR_CASE(128, 64)
  MLA_PAIR_CASE(192, 16) MLA_PAIR_CASE(192, 32) MLA_PAIR_CASE(192, 64)
#undef MLA_PAIR_CASE
  MLA_FAIL(MLA_ERR_UNSUPPORTED, "no pair attention kernel for d_c %d, d_rope %d", d.d_c, d.d_rope);
}

}  // namespace mla
