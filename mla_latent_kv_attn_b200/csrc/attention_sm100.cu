// attention_sm100.cu - latent-space multi-head attention of one chunk against the ring plus
// itself, on the sm_100a tensor cores (VideoMLA: hyper.ai summary, "Method": the score of head h
// adds q_nope.k_nope and q_rope.k_rope; keys/values are rebuilt from c_KV only when needed).
//
// In absorbed form every head is a query against the same keys K'_m = [c_m || RoPE(k_R,m)]
// (D = DC + DR wide) and the same values c_m (DC wide, the first DC columns of K'): MQA.
// The kernel is a template over the latent shape: DC in {128, 192, 256}, DR in {16, 32, 64}
// (the Wan preset is DC 192, DR 32: D 224); the figures below are for that shape.
//
// One CTA = one 128-row query tile of one head of one sample.  Roles (224 threads):
//   warps 0-3  softmax: one TMEM lane (= query row) per thread; online softmax in the log2
//              domain with lazy rescaling of O (only when the running max grows by > 8);
//              write P (bf16) into its TMEM buffer; final 1/l,
//              optional W_UV epilogue, stores and lse.
//              Before the loop they copy their query row into TMEM (DC <= 192, below).
//   warp 4     TMA producer: 128-key K' tiles into a 4-stage ring: three 128x64
//              (128B-swizzled) content blocks from the ring/chunk latents and one 128x32
//              (64B-swizzled) block of pre-rotated positional keys; then the W_UV_h tile.
//   warps 5, 6 TMEM allocation (warp 5); one thread of warp 5 issues the QK products, one of
//              warp 6 the PV products and the epilogue (two issuers keep the pipe fed):
//                S_j   = Q K'_j^T          M=128, N=128, K=224 (12 SW128 + 2 SW64 k-steps),
//                                          Q from TMEM
//                O    += P_j V_j           M=128, N=192, K=128; P from TMEM, V = content
//                                          blocks of the same stage read MN-major
//                o     = O_lat W_UV_h^T    M=128, N=128, K=192 (epilogue, O_lat bf16 in smem)
// TMEM columns: S [0,128), Q [128,128+D/2) as bf16 pairs, O [256,256+DC), P [256+DC,+64); the
// epilogue result reuses S.  With Q in TMEM the QK products read only K' from shared memory
// (with Q there too, its 4 KB per k-step doubled the operand traffic of QK), and the Q tile's
// shared memory holds a fourth K' stage.  One S buffer suffices: the softmax loads S(j) into
// registers and frees the buffer at once, so QK(j+1) overlaps the softmax of j; P has its own
// buffer for the same reason.
// With DC = 256 O and P leave no room for Q: Q stays in shared memory, there are two S buffers,
// P(j) is written into S buffer j&1 and QK(j+2) waits for PV(j).
#include "exp2.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace mla {

namespace {

using namespace sm100;

constexpr int kBM = 128;           // query rows per CTA
constexpr int kBN = kKeyTile;      // keys per tile
constexpr int kDh = 128;           // head width of the W_UV epilogue
constexpr int kSoftmaxThreads = 128;   // warps 0-3: one TMEM lane (query row) per thread
constexpr int kProducerWarp = 4;
constexpr int kQkWarp = 5;              // also allocates and frees TMEM
constexpr int kPvWarp = 6;
constexpr int kThreads = 224;

constexpr int kQBlk = kBM * 128;                 // 128 rows x 128 B: 16 KB (Q, O_lat, W_UV)
constexpr int kKBlk = kBN * 128;                 // 128 rows x 128 B: 16 KB (K' content)
constexpr int kSmemMax = 227 * 1024;             // dynamic shared memory a CTA may use
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 128;    // S buffers at columns 0 and 128
constexpr uint32_t kColO = 256;    // O: DC columns from here

// Layout of one latent shape: content width DC (a multiple of 64: DC/64 blocks of 128 rows x
// 128 B, 128-byte swizzle) and positional width DR (16, 32 or 64: one block of DR*2 bytes per
// row with the swizzle of that width).  The Q tile and every K' stage have this layout.
template <int DC_, int DR_>
struct AttnShape {
  static constexpr int DC = DC_, DR = DR_, D = DC + DR;
  static_assert(DC % 64 == 0 && DC >= 64 && DC <= 256, "DC must be 64, 128, 192 or 256");
  static_assert(DR == 16 || DR == 32 || DR == 64, "DR must be 16, 32 or 64");
  static constexpr int kCBlk = DC / 64;
  static constexpr int kRopeBytes = DR * 2;                // bytes per row of the rope block
  static constexpr uint32_t kRopeSwz = DR == 16 ? kSwizzle32B : DR == 32 ? kSwizzle64B
                                                                         : kSwizzle128B;
  static constexpr int kRopeSbo = 8 * kRopeBytes;          // one swizzle atom: 8 rows
  static constexpr int kRopeKSteps = DR / 16;
  static constexpr int kQTile = kCBlk * kQBlk + kBM * kRopeBytes;
  static constexpr int kKTile = kCBlk * kKBlk + kBN * kRopeBytes;
  // P (kBN/2 columns of packed bf16) gets its own TMEM columns after O when they fit; with a
  // 256-wide O it is written into the S buffer it came from instead.
  static constexpr bool kAliasP = kColO + DC + kBN / 2 > kTmemCols;
  static constexpr uint32_t kColP = kAliasP ? 0u : kColO + DC;
  // When P has its own columns, the query tile lives in TMEM (bf16 pairs, D/2 columns from
  // kColS, written by the softmax threads) in place of the second S buffer: QK reads only K'
  // from shared memory, and the tile's shared memory becomes one more K' stage.
  static constexpr bool kQTmem = !kAliasP && D / 2 <= 128;
  static constexpr int kQWords = (D / 2 + 15) / 16 * 16;    // TMEM columns written (zero tail)
  static constexpr int kQSmem = kQTmem ? 0 : kQTile;
  static constexpr int kFit = (kSmemMax - 1024 - kQSmem) / kKTile;
  static constexpr int kStages = kFit < 4 ? kFit : 4;
  // (with Q in TMEM, W_UV and O_lat take two different stages after the loop)
  static_assert(kStages >= (kQTmem ? 2 : 1), "too few K' stages fit in shared memory");
  static constexpr int kSmem = kQSmem + kStages * kKTile + 1024;
  static_assert(kKTile >= kCBlk * kQBlk, "the W_UV tile (and O_lat) go into K' stages");
};

struct AttnParams {
  const bf16* q;        // [B, n_q, H, D] (read by the softmax threads when Q lives in TMEM)
  int n_q, H, nc, nc_pad, nt_ring, nt;
  // Fused query heads: the K' ring first carries nqc chunk pairs (64 columns of the CTA's c_Q
  // rows and of w_qcat[h]); their product Q'_h accumulates in TMEM, and the softmax threads
  // rotate its positional part at (first_frame + n / tpf, row, column) and write Q as bf16.
  int nqc;
  int first_frame;
  RopeGeom rope;
  float scale_log2;
  int has_w_uv;
  void* out;
  float* lse;
  int32_t* dev_status;
};

// Pairs (out of every 8) of a full key tile whose exponentials take the FMA-pipe polynomial.
constexpr int kPolyPairsPer8 = 2;

// p = 2^(s * scale_log2 - m) for one row of a key tile: packed to bf16 pairs in w, returning
// the row sum.  kPoly: some pairs use exp2_poly_pair (full tiles; no masked -inf scores).
template <bool kPoly>
__device__ __forceinline__ float softmax_exp_row(const float (&s)[kKeyTile], float scale_log2,
                                                 float m, uint32_t (&w)[kKeyTile / 2]) {
  const uint64_t sc2 = f2_pack(scale_log2, scale_log2);
  const uint64_t nm2 = f2_pack(-m, -m);
  uint64_t sum2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
  for (int i = 0; i < kKeyTile / 2; ++i) {
    float x0, x1, p0, p1;
    f2_unpack(f2_fma(f2_pack(s[2 * i], s[2 * i + 1]), sc2, nm2), x0, x1);
    if (kPoly && (i & 7) < kPolyPairsPer8) {
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

// A query row into this thread's TMEM lane from column taddr on, as bf16 pairs (zeros past D/2
// and for row == nullptr).  All of the row's 16-byte pieces are loaded before the first store,
// so the row costs one global-load round trip instead of one per 16 columns.  Not inlined: with
// the unrolled loads in the kernel body the compiler's register allocation for the main loop
// changed and the kernel ran 3-4 % slower; as a separate function it is 1 % faster.
template <int D, int kQWords>
__device__ __noinline__ void copy_q_row(uint32_t taddr, const bf16* row) {
  const uint4* src = reinterpret_cast<const uint4*>(row);
  constexpr int kPieces = kQWords / 4;
  uint4 v[kPieces];
#pragma unroll
  for (int u = 0; u < kPieces; ++u)
    v[u] = src != nullptr && u < D / 8 ? src[u] : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
  for (int c = 0; c < kQWords; c += 16) {
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 x = v[c / 4 + i];
      w[4 * i] = x.x; w[4 * i + 1] = x.y; w[4 * i + 2] = x.z; w[4 * i + 3] = x.w;
    }
    tmem_st16(taddr + c, w);
  }
}

// Fused query heads: one row of Q'_h (fp32, TMEM columns kColO .. kColO+D of this thread's lane)
// rotated by 3D-RoPE in its last D-DC columns at chunk token n's position, rounded once to
// bf16 and stored as pairs from column kColS (zeros past D/2) - what the Q' GEMM's epilogue
// stores.  16 columns at a time: D is a multiple of 16 and DC of 64.
template <int DC>
__device__ __forceinline__ void q_piece(uint32_t tlane, int c, const AttnParams& p, int t, int hh,
                                        int ww, uint32_t* w8) {
  uint32_t r[16];
  tmem_ld16_wait(tlane + kColO + c, r);
  float v[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) v[k] = __uint_as_float(r[k]);
  if (c >= DC) {
#pragma unroll
    for (int k = 0; k < 16; k += 2)
      rope_rotate(v[k], v[k + 1], rope_angle(p.rope, (c - DC + k) >> 1, t, hh, ww));
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) w8[k] = pack_bf16x2(v[2 * k], v[2 * k + 1]);
}

template <int DC, int D, int kQWords>
__device__ __noinline__ void q_row_from_accumulator(uint32_t tlane, const AttnParams& p, int n) {
  const int nl = n < p.n_q ? n : 0;
  const int i = nl % p.rope.tpf;
  const int t = p.first_frame + nl / p.rope.tpf, hh = i / p.rope.frame_w, ww = i % p.rope.frame_w;
#pragma unroll 1
  for (int c = 0; c < kQWords * 2; c += 32) {     // 32 values = 16 bf16 pairs per store
    uint32_t w[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) w[k] = 0u;
    if (c < D) q_piece<DC>(tlane, c, p, t, hh, ww, w);
    if (c + 16 < D) q_piece<DC>(tlane, c + 16, p, t, hh, ww, w + 8);
    tmem_st16(tlane + kColS + c / 2, w);
  }
}

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                         int32_t* dev_status) {
  return mbar_wait_or_abort(bar, parity, abort_flag, dev_status);
}

template <int DC, int DR, bool kFusedQ>
__global__ void __launch_bounds__(kThreads, 1)
    attention_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_qr,
                        const __grid_constant__ CUtensorMap tm_cache,
                        const __grid_constant__ CUtensorMap tm_chunk,
                        const __grid_constant__ CUtensorMap tm_ws,
                        const __grid_constant__ CUtensorMap tm_wuv,
                        const __grid_constant__ CUtensorMap tm_cq,
                        const __grid_constant__ CUtensorMap tm_wq,
                        const __grid_constant__ AttnParams p) {
  using Sh = AttnShape<DC, DR>;
  constexpr int kDc = DC;
  constexpr int kCBlk = Sh::kCBlk;
  constexpr int kStages = Sh::kStages;
  constexpr int kQTile = Sh::kQTile;
  constexpr int kKTile = Sh::kKTile;
  constexpr bool kAliasP = Sh::kAliasP;
  constexpr uint32_t kColP = Sh::kColP;
  constexpr bool kQTmem = Sh::kQTmem;
  static_assert(!kFusedQ || kQTmem, "fused query heads need the query tile in TMEM");
  // a chunk pair of the fused query heads: 128 x 64 of c_Q, then D x 64 of w_qcat[h]
  constexpr int kCqBytes = kBM * 128, kWqBytes = Sh::D * 128;
  static_assert(!kFusedQ || kCqBytes + kWqBytes <= kKTile, "a query chunk pair fits a K' stage");
  const int nqc = kFusedQ ? p.nqc : 0;   // ring uses before the first K' tile
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t q_full;   // the Q tile landed (TMA) or is in TMEM (softmax)
  __shared__ __align__(8) uint64_t kv_full[kStages];
  __shared__ __align__(8) uint64_t kv_empty[kStages];
  __shared__ __align__(8) uint64_t s_full[2];
  __shared__ __align__(8) uint64_t s_free[2];
  __shared__ __align__(8) uint64_t p_full;
  __shared__ __align__(8) uint64_t pv_done;
  __shared__ __align__(8) uint64_t pv_buf_done[2];   // PV(j) done, per S buffer (aliased P)
  __shared__ __align__(8) uint64_t w_full;
  __shared__ __align__(8) uint64_t olat_full;
  __shared__ __align__(8) uint64_t epi_done;
  __shared__ __align__(8) uint64_t qacc_full;   // fused query heads: Q'_h accumulated in TMEM
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sQ = sbase;                     // (the Q tile, when it is in shared memory)
  const uint32_t sK0 = sbase + Sh::kQSmem;       // K' stage 0
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int q0 = qt * kBM;
  volatile int* abort_flag = &abort_sh;

  if (threadIdx.x == 0) {
    abort_sh = 0;
    mbar_init(smem_u32(&q_full), kQTmem ? kSoftmaxThreads : 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&kv_full[s]), 1);
      mbar_init(smem_u32(&kv_empty[s]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&s_full[i]), 1);
      mbar_init(smem_u32(&s_free[i]), kSoftmaxThreads);
    }
    mbar_init(smem_u32(&p_full), kSoftmaxThreads);
    mbar_init(smem_u32(&pv_done), 1);
    mbar_init(smem_u32(&pv_buf_done[0]), 1);
    mbar_init(smem_u32(&pv_buf_done[1]), 1);
    mbar_init(smem_u32(&w_full), 1);
    mbar_init(smem_u32(&olat_full), kSoftmaxThreads);
    mbar_init(smem_u32(&epi_done), 1);
    mbar_init(smem_u32(&qacc_full), 1);

    fence_barrier_init();
  }
  if (warp == kQkWarp) {
    tmem_alloc(smem_u32(&tmem_base_sh), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  // launched with programmatic serialisation: the set-up above may overlap the previous
  // kernel's tail; nothing global is touched before it has completed
  grid_dep_wait();
  grid_dep_launch();

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_chunk);
      tma_prefetch_desc(&tm_ws);
      if constexpr (!kQTmem) {
        tma_prefetch_desc(&tm_q);
        const uint32_t qb = smem_u32(&q_full);
        mbar_arrive_expect_tx(qb, kQTile);
        for (int i = 0; i < kCBlk; ++i) tma_load_4d(sQ + i * kQBlk, &tm_q, qb, 64 * i, h, q0, b);
        tma_load_4d(sQ + kCBlk * kQBlk, &tm_qr, qb, kDc, h, q0, b);
      }
      bool ok = true;
      if constexpr (kFusedQ) {
        // the query heads' operands first: chunk c = columns 64c.. of c_Q rows q0.. and of
        // w_qcat[h] (its D rows), through the ring like K' tiles
        tma_prefetch_desc(&tm_cq);
        tma_prefetch_desc(&tm_wq);
        for (int c = 0; c < nqc && ok; ++c) {
          const int s = c % kStages;
          ok = wait_bar(smem_u32(&kv_empty[s]), ((c / kStages) & 1) ^ 1, abort_flag, p.dev_status);
          if (!ok) break;
          const uint32_t dst = sK0 + s * kKTile;
          const uint32_t fb = smem_u32(&kv_full[s]);
          mbar_arrive_expect_tx(fb, kCqBytes + kWqBytes);
          tma_load_3d(dst, &tm_cq, fb, 64 * c, q0, b);
          tma_load_2d(dst + kCqBytes, &tm_wq, fb, 64 * c, h * Sh::D);
        }
      }
      for (int j = 0; j < p.nt && ok; ++j) {
        const int u = nqc + j;                 // ring use of K' tile j
        const int s = u % kStages;
        ok = wait_bar(smem_u32(&kv_empty[s]), ((u / kStages) & 1) ^ 1, abort_flag, p.dev_status);
        if (!ok) break;
        const uint32_t dst = sK0 + s * kKTile;
        const uint32_t fb = smem_u32(&kv_full[s]);
        mbar_arrive_expect_tx(fb, kKTile);
        if (j < p.nt_ring) {
          const int r0 = j * kBN;
          for (int i = 0; i < kCBlk; ++i) tma_load_3d(dst + i * kKBlk, &tm_cache, fb, 64 * i, r0, b);
          tma_load_3d(dst + kCBlk * kKBlk, &tm_ws, fb, 0, r0, b);
        } else {
          const int r0 = (j - p.nt_ring) * kBN;
          for (int i = 0; i < kCBlk; ++i) tma_load_3d(dst + i * kKBlk, &tm_chunk, fb, 64 * i, r0, b);
          tma_load_3d(dst + kCBlk * kKBlk, &tm_ws, fb, 0, p.nc_pad + r0, b);
        }
      }
      if (ok && p.has_w_uv) {
        // W_UV_h [128 x DC] goes into the stage a tile nt would use, once it is free.
        const int uw = nqc + p.nt;
        const int s = uw % kStages;
        if (wait_bar(smem_u32(&kv_empty[s]), ((uw / kStages) & 1) ^ 1, abort_flag, p.dev_status)) {
          const uint32_t wb = smem_u32(&w_full);
          mbar_arrive_expect_tx(wb, kCBlk * kQBlk);
          for (int i = 0; i < kCBlk; ++i)
            tma_load_2d(sK0 + s * kKTile + i * kQBlk, &tm_wuv, wb, 64 * i, h * kDh);
        }
      }
    }
  } else if (warp == kQkWarp || warp == kPvWarp) {
    // ------------------------------------------------------------------ MMA issuers
    // Two threads issue MMAs: one the QK products, the other the PV products and the W_UV
    // epilogue.  A tcgen05.mma issue takes about as long as the tensor pipe needs to start
    // it, so the pipe only stays busy if some thread is always issuing; with two issuers one
    // waits on a barrier while the other feeds the pipe.  Order between the two streams is
    // explicit: QK(j) overwrites the S/P buffer that PV(j-2) reads, so it waits for PV(j-2).
    // With Q in TMEM there is one S buffer, which QK(j) takes once the softmax has loaded S(j-1).
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBM, kDc, 0, 1);
      constexpr uint32_t idesc_uv = idesc_bf16_f32(kBM, kDh, 0, 0);
      // Descriptors are built once; an operand at byte offset `off` from a descriptor's start
      // is that descriptor plus off/16 (the start-address field is the low 14 bits and every
      // address stays below 256 KB, so the add never carries out of the field).
      constexpr uint32_t kQBlkD = kQBlk >> 4, kKBlkD = kKBlk >> 4, kKTileD = kKTile >> 4;
      const uint64_t q_c = smem_desc(sQ, 16, 1024, kSwizzle128B);
      const uint64_t q_r = smem_desc(sQ + kCBlk * kQBlk, 16, Sh::kRopeSbo, Sh::kRopeSwz);
      const uint64_t k_c0 = smem_desc(sK0, 16, 1024, kSwizzle128B);
      const uint64_t k_r0 = smem_desc(sK0 + kCBlk * kKBlk, 16, Sh::kRopeSbo, Sh::kRopeSwz);
      const uint64_t v_0 = smem_desc(sK0, kKBlk, 1024, kSwizzle128B);
      bool ok = true;
      if (warp == kQkWarp) {
        if constexpr (kFusedQ) {
          // Q'_h = c_Q rows x w_qcat[h]^T (M=128, N=D, K=d_cq) into TMEM columns kColO.. (free
          // until the first PV), then handed to the softmax threads
          constexpr uint32_t idesc_q = idesc_bf16_f32(kBM, Sh::D, 0, 0);
          for (int c = 0; c < nqc && ok; ++c) {
            const int s = c % kStages;
            ok = wait_bar(smem_u32(&kv_full[s]), (c / kStages) & 1, abort_flag, p.dev_status);
            if (!ok) break;
            tc_fence_after();
            const uint64_t a0 = smem_desc(sK0 + s * kKTile, 16, 1024, kSwizzle128B);
            const uint64_t b0 = smem_desc(sK0 + s * kKTile + kCqBytes, 16, 1024, kSwizzle128B);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ss(tmem + kColO, a0 + 2 * kk, b0 + 2 * kk, idesc_q, (c | kk) != 0 ? 1u : 0u);
            mma_commit(smem_u32(&kv_empty[s]));
          }
          if (ok) mma_commit(smem_u32(&qacc_full));
        }
        ok = ok && wait_bar(smem_u32(&q_full), 0, abort_flag, p.dev_status);
        for (int j = 0; j < p.nt && ok; ++j) {
          const int u = nqc + j;
          const int s = u % kStages;
          ok = wait_bar(smem_u32(&kv_full[s]), (u / kStages) & 1, abort_flag, p.dev_status);
          if constexpr (kQTmem) {    // the softmax has loaded S(j-1) out of the one buffer
            if (ok && j >= 1)
              ok = wait_bar(smem_u32(&s_free[0]), (j - 1) & 1, abort_flag, p.dev_status);
          } else if (ok && j >= 2) {
            if constexpr (kAliasP)   // PV(j-2) has read P(j-2) out of the buffer this QK overwrites
              ok = wait_bar(smem_u32(&pv_buf_done[j & 1]), ((j - 2) >> 1) & 1, abort_flag,
                            p.dev_status);
            else                     // the softmax has loaded S(j-2) out of that buffer
              ok = wait_bar(smem_u32(&s_free[j & 1]), ((j - 2) >> 1) & 1, abort_flag, p.dev_status);
          }
          if (!ok) break;
          tc_fence_after();
          const uint64_t kc = k_c0 + static_cast<uint32_t>(s) * kKTileD;
          const uint64_t kr = k_r0 + static_cast<uint32_t>(s) * kKTileD;
          if constexpr (kQTmem) {
            // A = Q from TMEM: 8 columns (16 bf16) per k-step, content then positional
            const uint32_t qa = tmem + kColS;
#pragma unroll
            for (int blk = 0; blk < kCBlk; ++blk)
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_ts(tmem, qa + 8 * (4 * blk + kk), kc + (blk * kKBlkD + 2 * kk), idesc_qk,
                       (blk | kk) != 0 ? 1u : 0u);
#pragma unroll
            for (int kk = 0; kk < Sh::kRopeKSteps; ++kk)
              mma_ts(tmem, qa + 8 * (4 * kCBlk + kk), kr + 2 * kk, idesc_qk, 1u);
            mma_commit(smem_u32(&s_full[0]));
          } else {
            const uint32_t d = tmem + (j & 1) * kColS;
#pragma unroll
            for (int blk = 0; blk < kCBlk; ++blk)
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_ss(d, q_c + (blk * kQBlkD + 2 * kk), kc + (blk * kKBlkD + 2 * kk), idesc_qk,
                       (blk | kk) != 0 ? 1u : 0u);
#pragma unroll
            for (int kk = 0; kk < Sh::kRopeKSteps; ++kk)
              mma_ss(d, q_r + 2 * kk, kr + 2 * kk, idesc_qk, 1u);
            mma_commit(smem_u32(&s_full[j & 1]));
          }
        }
      } else {
        for (int j = 0; j < p.nt && ok; ++j) {
          ok = wait_bar(smem_u32(&p_full), j & 1, abort_flag, p.dev_status);
          if (!ok) break;
          tc_fence_after();
          const int s = (nqc + j) % kStages;
          const uint64_t vd = v_0 + static_cast<uint32_t>(s) * kKTileD;
          const uint32_t pa = tmem + (kAliasP ? (j & 1) * kColS : kColP);
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk)
            // V rows kk*16 .. +15: 16 rows of 128 B further per step (2048 B = 128 units)
            mma_ts(tmem + kColO, pa + kk * 8, vd + 128 * kk, idesc_pv, (j | kk) != 0 ? 1u : 0u);
          mma_commit(smem_u32(&kv_empty[s]));
          mma_commit(smem_u32(&pv_done));
          if constexpr (kAliasP) mma_commit(smem_u32(&pv_buf_done[j & 1]));
        }
        if (ok && p.has_w_uv) {
          ok = wait_bar(smem_u32(&w_full), 0, abort_flag, p.dev_status) &&
               wait_bar(smem_u32(&olat_full), 0, abort_flag, p.dev_status);
          if (ok) {
            tc_fence_after();
            const uint64_t w_c = smem_desc(sK0 + ((nqc + p.nt) % kStages) * kKTile, 16, 1024,
                                           kSwizzle128B);
            // O_lat: in the dead Q tile, or (Q in TMEM) in the stage after W_UV's
            const uint64_t o_c =
                kQTmem ? smem_desc(sK0 + ((nqc + p.nt + 1) % kStages) * kKTile, 16, 1024, kSwizzle128B)
                       : q_c;
#pragma unroll
            for (int blk = 0; blk < kCBlk; ++blk)
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_ss(tmem, o_c + (blk * kQBlkD + 2 * kk), w_c + (blk * kQBlkD + 2 * kk), idesc_uv,
                       (blk | kk) != 0 ? 1u : 0u);
            mma_commit(smem_u32(&epi_done));
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax warps 0..3
    const int row = warp * 32 + lane;                 // TMEM lane and query row in the tile
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const int n = q0 + row;
    if constexpr (kFusedQ) {
      // this row of Q'_h out of its fp32 accumulator, the positional part rotated at the row's
      // position, into the query's TMEM columns as bf16 pairs
      const bool okq = __all_sync(0xffffffffu, wait_bar(smem_u32(&qacc_full), 0, abort_flag,
                                                        p.dev_status));
      if (okq) {
        tc_fence_after();
        q_row_from_accumulator<DC, Sh::D, Sh::kQWords>(tmem + lane_off, p, n);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(smem_u32(&q_full));
    } else if constexpr (kQTmem) {
      // this row of the query tile into TMEM, bf16 pairs from column kColS (zeros past D/2
      // and for rows past n_q); the QK issuer waits for all 128 rows on q_full
      copy_q_row<Sh::D, Sh::kQWords>(tmem + lane_off + kColS,
                                     n < p.n_q ? p.q + ((static_cast<int64_t>(b) * p.n_q + n) * p.H + h) * Sh::D
                                               : nullptr);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(smem_u32(&q_full));
    }
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < p.nt; ++j) {
      // S buffer and phase: one buffer with Q in TMEM, else two used in turn
      const int sb = kQTmem ? 0 : (j & 1);
      const uint32_t sphase = kQTmem ? (j & 1) : ((j >> 1) & 1);
      ok = __all_sync(0xffffffffu,
                      wait_bar(smem_u32(&s_full[sb]), sphase, abort_flag, p.dev_status));
      if (!ok) break;
      tc_fence_after();
      float s[kBN];
      {
        uint32_t r[kBN];
        tmem_ld128_wait(tmem + lane_off + sb * kColS, r);
#pragma unroll
        for (int i = 0; i < kBN; ++i) s[i] = __uint_as_float(r[i]);
      }
      const int valid = j < p.nt_ring ? min(kBN, p.nc - j * kBN)
                                      : min(kBN, p.n_q - (j - p.nt_ring) * kBN);
      if (valid < kBN) {                    // only the last tile of the ring or of the chunk
#pragma unroll
        for (int c = 0; c < kBN; ++c)
          if (c >= valid) s[c] = -INFINITY;
      }
      // Row max of the raw scores (the scale is positive): eight independent chains of
      // three-input maxima, chain u covering columns u, u+8, ..., u+120.
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
      // S(j) is in registers: its TMEM buffer may take the next QK (with P in its own buffer;
      // an aliased P keeps the buffer until PV(j) has read it).  Released after the row max,
      // not right after the load: the QK issuer's MMAs then do not compete with the max for
      // the issue slots of the sub-partitions it shares with softmax warps (measured: the call
      // 1.1 % shorter).
      if constexpr (!kAliasP) {
        tc_fence_before();
        mbar_arrive(smem_u32(&s_free[sb]));
      }
      // Lazy rescaling: the running max moves only when a row's max grows by more than 8
      // (a factor 256), so p stays below 256 and O is rescaled rarely.
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
      // p = 2^(s * scale * log2(e) - m): one packed FFMA2 per two scores, then ex2 on the MUFU
      // unit or, for a fixed share of the pairs of full tiles, the FMA-pipe polynomial; packed
      // to bf16 pairs; the row sum runs in four packed FADD2 chains.
      uint32_t w[kBN / 2];
      if (valid == kBN) l_run += softmax_exp_row<true>(s, p.scale_log2, m_run, w);
      else l_run += softmax_exp_row<false>(s, p.scale_log2, m_run, w);
      // The P buffer and O are free once PV(j-1) has completed (an aliased P needs only O).
      if (j > 0 && (!kAliasP || rescale)) {
        ok = __all_sync(0xffffffffu,
                        wait_bar(smem_u32(&pv_done), (j - 1) & 1, abort_flag, p.dev_status));
        if (!ok) break;
        tc_fence_after();
      }
      if (rescale) {
#pragma unroll 1
        for (int c = 0; c < kDc; c += 16) {
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
        tmem_st16(tmem + lane_off + (kAliasP ? (j & 1) * kColS : kColP) + c, w16);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(smem_u32(&p_full));
    }
    if (ok)
      ok = __all_sync(0xffffffffu,
                      wait_bar(smem_u32(&pv_done), (p.nt - 1) & 1, abort_flag, p.dev_status));
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.f / l_run;
      if (p.lse != nullptr && n < p.n_q)
        p.lse[(static_cast<int64_t>(b) * p.H + h) * p.n_q + n] =
            (m_run + log2f(l_run)) * 0.69314718055994530942f;
      if (!p.has_w_uv) {
        bf16* orow = static_cast<bf16*>(p.out) +
                     ((static_cast<int64_t>(b) * p.n_q + n) * p.H + h) * kDc;
#pragma unroll 1
        for (int c = 0; c < kDc; c += 32) {
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
        // O_lat (bf16) -> shared memory, 128B-swizzled K-major, over the dead Q tile (or, with
        // Q in TMEM, into the K' stage after the one W_UV went to: all stages are free now).
        const uint32_t so = kQTmem ? sK0 + ((nqc + p.nt + 1) % kStages) * kKTile : sQ;
        uint8_t* qsm = smem_raw + (so - smem_u32(smem_raw));
#pragma unroll 1
        for (int c = 0; c < kDc; c += 32) {
          uint32_t r[32];
          tmem_ld32_wait(tmem + lane_off + kColO + c, r);
          const int blk = c / 64;
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {         // four 16-byte chunks of 8 values
            const int chunk = (c % 64) / 8 + ch;   // chunk index within the 128-byte row
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(r[8 * ch + 0]) * inv_l, __uint_as_float(r[8 * ch + 1]) * inv_l);
            v.y = pack_bf16x2(__uint_as_float(r[8 * ch + 2]) * inv_l, __uint_as_float(r[8 * ch + 3]) * inv_l);
            v.z = pack_bf16x2(__uint_as_float(r[8 * ch + 4]) * inv_l, __uint_as_float(r[8 * ch + 5]) * inv_l);
            v.w = pack_bf16x2(__uint_as_float(r[8 * ch + 6]) * inv_l, __uint_as_float(r[8 * ch + 7]) * inv_l);
            const int off = blk * kQBlk + row * 128 + ((chunk ^ (row & 7)) * 16);
            *reinterpret_cast<uint4*>(qsm + off) = v;
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(smem_u32(&olat_full));
        ok = __all_sync(0xffffffffu, wait_bar(smem_u32(&epi_done), 0, abort_flag, p.dev_status));
        if (ok) {
          tc_fence_after();
          bf16* orow = static_cast<bf16*>(p.out) +
                       (static_cast<int64_t>(b) * p.n_q + n) * (static_cast<int64_t>(p.H) * kDh) +
                       static_cast<int64_t>(h) * kDh;
#pragma unroll 1
          for (int c = 0; c < kDh; c += 32) {
            uint32_t r[32];
            tmem_ld32_wait(tmem + lane_off + c, r);
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
  if (warp == kQkWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Fused query heads (attention_tc_fused_q): c_q [B, n_q, d_cq] and w_qcat [H, D, d_cq] in place
// of a.q, and the chunk's first frame for the query's 3D-RoPE.
struct FusedQ {
  const void* c_q;
  const void* w_qcat;
  int first_frame;
};

template <int DC, int DR, bool kFusedQ>
mla_status attention_tc_impl(const Dims& d, const AttnArgs& a, int n_valid, cudaStream_t s,
                             const FusedQ* fq = nullptr) {
  using Sh = AttnShape<DC, DR>;
  constexpr int kD = Sh::D;
  const KeyWorkspace kw = key_workspace_layout(d, n_valid);
  CUtensorMap tq, tqr, tcache, tchunk, tws, twuv, tcq, twq;
  mla_status st;
  if (kFusedQ) {
    const uint64_t dims[3] = {static_cast<uint64_t>(d.d_cq), static_cast<uint64_t>(d.n_q),
                              static_cast<uint64_t>(d.B)};
    const uint64_t strides[2] = {static_cast<uint64_t>(d.d_cq) * 2,
                                 static_cast<uint64_t>(d.n_q) * d.d_cq * 2};
    const uint32_t box[3] = {64, kBM, 1};
    if ((st = make_tmap_bf16(&tcq, fq->c_q, 3, dims, strides, box, 128)) != MLA_OK) return st;
    const uint64_t wdims[2] = {static_cast<uint64_t>(d.d_cq), static_cast<uint64_t>(d.H) * kD};
    const uint64_t wstrides[1] = {static_cast<uint64_t>(d.d_cq) * 2};
    const uint32_t wbox[2] = {64, kD};
    if ((st = make_tmap_bf16(&twq, fq->w_qcat, 2, wdims, wstrides, wbox, 128)) != MLA_OK) return st;
    tq = tcq;    // never read: the query comes from the fused heads
    tqr = tcq;
  } else {
    const uint64_t dims[4] = {static_cast<uint64_t>(kD), static_cast<uint64_t>(d.H),
                              static_cast<uint64_t>(d.n_q), static_cast<uint64_t>(d.B)};
    const uint64_t strides[3] = {kD * 2ull, static_cast<uint64_t>(d.H) * kD * 2,
                                 static_cast<uint64_t>(d.n_q) * d.H * kD * 2};
    const uint32_t box[4] = {64, 1, kBM, 1};
    if ((st = make_tmap_bf16(&tq, a.q, 4, dims, strides, box, 128)) != MLA_OK) return st;
    const uint32_t box_r[4] = {DR, 1, kBM, 1};
    if ((st = make_tmap_bf16(&tqr, a.q, 4, dims, strides, box_r, Sh::kRopeBytes)) != MLA_OK)
      return st;
    tcq = tq;    // never read
    twq = tq;
  }
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(kD), static_cast<uint64_t>(d.n_q),
                              static_cast<uint64_t>(d.B)};
    const uint64_t strides[2] = {kD * 2ull, static_cast<uint64_t>(d.n_q) * kD * 2};
    const uint32_t box[3] = {64, kBN, 1};
    if ((st = make_tmap_bf16(&tchunk, a.chunk_lat, 3, dims, strides, box, 128)) != MLA_OK) return st;
  }
  if (kw.nc > 0) {
    const uint64_t dims[3] = {static_cast<uint64_t>(kD), static_cast<uint64_t>(kw.nc),
                              static_cast<uint64_t>(d.B)};
    const uint64_t strides[2] = {kD * 2ull, static_cast<uint64_t>(d.W) * d.tpf * kD * 2};
    const uint32_t box[3] = {64, kBN, 1};
    if ((st = make_tmap_bf16(&tcache, a.cache, 3, dims, strides, box, 128)) != MLA_OK) return st;
  } else {
    tcache = tchunk;  // never read: no ring tiles
  }
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(DR), static_cast<uint64_t>(kw.rows),
                              static_cast<uint64_t>(d.B)};
    const uint64_t strides[2] = {DR * 2ull, static_cast<uint64_t>(kw.rows) * DR * 2};
    const uint32_t box[3] = {DR, kBN, 1};
    if ((st = make_tmap_bf16(&tws, a.ws, 3, dims, strides, box, Sh::kRopeBytes)) != MLA_OK)
      return st;
  }
  if (a.w_uv != nullptr) {
    const uint64_t dims[2] = {static_cast<uint64_t>(DC), static_cast<uint64_t>(d.H) * kDh};
    const uint64_t strides[1] = {DC * 2ull};
    const uint32_t box[2] = {64, kDh};
    if ((st = make_tmap_bf16(&twuv, a.w_uv, 2, dims, strides, box, 128)) != MLA_OK) return st;
  } else {
    twuv = tchunk;    // never read
  }
  AttnParams p;
  p.q = static_cast<const bf16*>(a.q);
  p.n_q = d.n_q; p.H = d.H; p.nc = kw.nc; p.nc_pad = kw.nc_pad;
  p.nt_ring = ceil_div(kw.nc, kBN);
  p.nt = p.nt_ring + ceil_div(d.n_q, kBN);
  p.scale_log2 = d.scale * 1.4426950408889634f;
  p.has_w_uv = a.w_uv != nullptr;
  p.out = a.out; p.lse = a.lse; p.dev_status = a.dev_status;
  p.nqc = kFusedQ ? d.d_cq / 64 : 0;
  p.first_frame = kFusedQ ? fq->first_frame : 0;
  p.rope = rope_geom(d);
  MLA_CUDA_TRY(cudaFuncSetAttribute(attention_tc_kernel<DC, DR, kFusedQ>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, Sh::kSmem));
  dim3 grid(ceil_div(d.n_q, kBM), d.H, d.B);
  MLA_CUDA_TRY(launch_pdl(attention_tc_kernel<DC, DR, kFusedQ>, grid, dim3(kThreads), Sh::kSmem,
                          s, tq, tqr, tcache, tchunk, tws, twuv, tcq, twq, p));
  MLA_LAUNCH_CHECK("attention_tc");
  return MLA_OK;
}

}  // namespace

bool tc_attention_supported(const Dims& d, bool has_w_uv) {
  return d.dtype == MLA_BF16 && (d.d_c == 128 || d.d_c == 192 || d.d_c == 256) &&
         (d.d_rope == 16 || d.d_rope == 32 || d.d_rope == 64) && (!has_w_uv || d.d_head == kDh);
}

mla_status attention_tc(const Dims& d, const AttnArgs& a, int n_valid, cudaStream_t s) {
#define MLA_ATTN_CASE(DC, DR) \
  if (d.d_c == DC && d.d_rope == DR) return attention_tc_impl<DC, DR, false>(d, a, n_valid, s);
  MLA_ATTN_CASE(128, 16) MLA_ATTN_CASE(128, 32) MLA_ATTN_CASE(128, 64)
  MLA_ATTN_CASE(192, 16) MLA_ATTN_CASE(192, 32) MLA_ATTN_CASE(192, 64)
  MLA_ATTN_CASE(256, 16) MLA_ATTN_CASE(256, 32) MLA_ATTN_CASE(256, 64)
#undef MLA_ATTN_CASE
  MLA_FAIL(MLA_ERR_UNSUPPORTED, "no tensor-core attention kernel for d_c %d, d_rope %d", d.d_c,
           d.d_rope);
}

bool tc_attention_fused_q_supported(const Dims& d, bool has_w_uv) {
  return tc_attention_supported(d, has_w_uv) && d.d_c <= 192 && d.d_c + d.d_rope <= 256 &&
         d.d_cq % 64 == 0 && d.d_cq > 0;
}

mla_status attention_tc_fused_q(const Dims& d, const AttnArgs& a, int n_valid, const void* c_q,
                                const void* w_qcat, int first_frame, cudaStream_t s) {
  const FusedQ fq{c_q, w_qcat, first_frame};
#define MLA_ATTN_FQ_CASE(DC, DR) \
  if (d.d_c == DC && d.d_rope == DR) return attention_tc_impl<DC, DR, true>(d, a, n_valid, s, &fq);
  MLA_ATTN_FQ_CASE(128, 16) MLA_ATTN_FQ_CASE(128, 32) MLA_ATTN_FQ_CASE(128, 64)
  MLA_ATTN_FQ_CASE(192, 16) MLA_ATTN_FQ_CASE(192, 32) MLA_ATTN_FQ_CASE(192, 64)
#undef MLA_ATTN_FQ_CASE
  MLA_FAIL(MLA_ERR_UNSUPPORTED, "no fused-query attention kernel for d_c %d, d_rope %d", d.d_c,
           d.d_rope);
}

}  // namespace mla
