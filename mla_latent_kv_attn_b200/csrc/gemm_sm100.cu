// gemm_sm100.cu - bf16 GEMM on the 5th-generation tensor cores for the projections of the
// path (KV down-projection, query latent, absorbed query heads, value up-projection, W_O).
//
//   C[z](m, n) = sum_k A[z](m, k) * B[z](n, k)     bf16 operands, fp32 accumulation in TMEM
//
// One CTA computes a 128 x BN tile.  Warp 0 streams 128x64 (A) and BNx64 (B) K-slices into a
// 4-stage ring of 128B-swizzled shared-memory buffers with TMA; warp 1 allocates TMEM and one of
// its threads issues tcgen05.mma (M=128, N=BN, K=16 per instruction) and commits each stage
// back to the producer; warps 2..5 drain the fp32 accumulator from TMEM (one lane = one row),
// optionally rotate the positional-query columns (3D-RoPE), and store bf16 rows.
#include "kernels.h"
#include "sm100.cuh"

namespace mla {

namespace {

using namespace sm100;

constexpr int kBM = 128;
constexpr int kBK = 64;          // one 128-byte swizzle atom of bf16 per row
constexpr int kStages = 4;
constexpr int kThreads = 192;    // 6 warps

template <int BN>
struct GemmCfg {
  static constexpr int kATile = kBM * kBK * 2;
  static constexpr int kBTile = BN * kBK * 2;
  static constexpr int kStage = kATile + kBTile;
  static constexpr int kSmem = kStages * kStage + 1024;  // + slack to align to 1024 B
  static constexpr int kTmemCols = BN <= 32 ? 32 : BN <= 64 ? 64 : BN <= 128 ? 128 : 256;
};

struct GemmParams {
  int M, N, K;
  int a_swapped, b_swapped;  // tensor map dims are (K, batch, rows) instead of (K, rows, batch)
  void* C;
  int64_t c_sm, c_batch;
  int epilogue;
  int rope_D, rope_n_q, rope_first_frame;
  RopeGeom rope;
};

__device__ __forceinline__ void store_row32(bf16* dst, const float* v, int valid, bool vec_ok) {
  if (vec_ok && valid >= 32) {
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) w[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
    uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int i = 0; i < 4; ++i) d4[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
  } else {
    for (int i = 0; i < valid && i < 32; ++i) dst[i] = __float2bfloat16_rn(v[i]);
  }
}

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   GemmParams p) {
  using Cfg = GemmCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[kStages];
  __shared__ __align__(8) uint64_t empty_bar[kStages];
  __shared__ __align__(8) uint64_t acc_bar;
  __shared__ uint32_t tmem_base_sh;

  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n0 = blockIdx.x * BN, m0 = blockIdx.y * kBM, z = blockIdx.z;
  const int nkb = ceil_div(p.K, kBK);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    mbar_init(smem_u32(&acc_bar), 1);
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

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % kStages;
        const uint32_t ph = (kb / kStages) & 1;
        if (!mbar_wait(smem_u32(&empty_bar[s]), ph ^ 1)) break;
        const uint32_t a_dst = base + s * Cfg::kStage;
        const uint32_t b_dst = a_dst + Cfg::kATile;
        const uint32_t fb = smem_u32(&full_bar[s]);
        mbar_arrive_expect_tx(fb, Cfg::kStage);
        if (p.a_swapped) tma_load_3d(a_dst, &tmA, fb, kb * kBK, z, m0);
        else tma_load_3d(a_dst, &tmA, fb, kb * kBK, m0, z);
        if (p.b_swapped) tma_load_3d(b_dst, &tmB, fb, kb * kBK, z, n0);
        else tma_load_3d(b_dst, &tmB, fb, kb * kBK, n0, z);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kBM, BN, 0, 0);
      bool ok = true;
      for (int kb = 0; kb < nkb && ok; ++kb) {
        const int s = kb % kStages;
        const uint32_t ph = (kb / kStages) & 1;
        ok = mbar_wait(smem_u32(&full_bar[s]), ph);
        if (!ok) break;
        tc_fence_after();
        const uint32_t a_addr = base + s * Cfg::kStage;
        const uint32_t b_addr = a_addr + Cfg::kATile;
#pragma unroll
        for (int k = 0; k < kBK / 16; ++k) {
          const uint64_t ad = smem_desc(a_addr + 32 * k, 16, 1024, kSwizzle128B);
          const uint64_t bd = smem_desc(b_addr + 32 * k, 16, 1024, kSwizzle128B);
          mma_ss(tmem, ad, bd, idesc, (kb | k) != 0 ? 1u : 0u);
        }
        mma_commit(smem_u32(&empty_bar[s]));
      }
      if (ok) mma_commit(smem_u32(&acc_bar));
    }
  } else {
    // epilogue warps 2..5 cover TMEM lane quadrants 2, 3, 0, 1
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const int m = m0 + row;
    const bool ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&acc_bar), 0));
    tc_fence_after();
    if (ok) {
      bf16* crow = static_cast<bf16*>(p.C) + static_cast<int64_t>(z) * p.c_batch +
                   static_cast<int64_t>(m) * p.c_sm;
      const bool vec_ok = ((reinterpret_cast<uintptr_t>(p.C) & 15u) == 0) && (p.c_sm % 8 == 0) &&
                          (p.c_batch % 8 == 0);
      int t = 0, hh = 0, ww = 0;
      if (p.epilogue == kEpiRopeQ) {
        const int nl = m % p.rope_n_q;
        const int i = nl % p.rope.tpf;
        t = p.rope_first_frame + nl / p.rope.tpf;
        hh = i / p.rope.frame_w;
        ww = i % p.rope.frame_w;
      }
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t r[32];
        tmem_ld32_wait(tmem + (static_cast<uint32_t>(quad * 32) << 16) + c0, r);
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
        if (p.epilogue == kEpiRopeQ && ((n0 + c0) % p.rope_D) == p.rope_D - 32) {
#pragma unroll
          for (int pr = 0; pr < 16; ++pr)
            rope_rotate(v[2 * pr], v[2 * pr + 1], rope_angle(p.rope, pr, t, hh, ww));
        }
        const int n = n0 + c0;
        if (m < p.M && n < p.N) store_row32(crow + n, v, p.N - n, vec_ok);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

// Tensor map over one operand [batch][rows, K] (K contiguous).  TMA wants increasing strides,
// so when the batch stride is below the row stride the map is built over (K, batch, rows).
mla_status operand_map(CUtensorMap* map, const void* base, int K, int rows, int batch,
                       int64_t row_stride, int64_t batch_stride, uint32_t box_rows, int* swapped) {
  const int64_t bs = batch > 1 ? batch_stride : row_stride * rows;
  *swapped = (batch > 1 && bs < row_stride) ? 1 : 0;
  if (*swapped) {
    const uint64_t dims[3] = {static_cast<uint64_t>(K), static_cast<uint64_t>(batch),
                              static_cast<uint64_t>(rows)};
    const uint64_t strides[2] = {static_cast<uint64_t>(bs) * 2, static_cast<uint64_t>(row_stride) * 2};
    const uint32_t box[3] = {static_cast<uint32_t>(kBK), 1, box_rows};
    return make_tmap_bf16(map, base, 3, dims, strides, box, 128);
  }
  const uint64_t dims[3] = {static_cast<uint64_t>(K), static_cast<uint64_t>(rows),
                            static_cast<uint64_t>(batch)};
  const uint64_t strides[2] = {static_cast<uint64_t>(row_stride) * 2, static_cast<uint64_t>(bs) * 2};
  const uint32_t box[3] = {static_cast<uint32_t>(kBK), box_rows, 1};
  return make_tmap_bf16(map, base, 3, dims, strides, box, 128);
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
  p.M = g.M; p.N = g.N; p.K = g.K; p.a_swapped = a_sw; p.b_swapped = b_sw; p.C = g.C; p.c_sm = g.c_sm; p.c_batch = g.c_batch;
  p.epilogue = g.epilogue; p.rope_D = g.rope_D; p.rope_n_q = g.rope_n_q;
  p.rope_first_frame = g.rope_first_frame; p.rope = g.rope;
  MLA_CUDA_TRY(cudaFuncSetAttribute(gemm_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    Cfg::kSmem));
  dim3 grid(ceil_div(g.N, BN), ceil_div(g.M, kBM), g.batch);
  gemm_tc_kernel<BN><<<grid, kThreads, Cfg::kSmem, s>>>(ta, tb, p);
  MLA_LAUNCH_CHECK("gemm_tc");
  return MLA_OK;
}

}  // namespace

bool tc_gemm_supported(int M, int N, int K, int64_t a_sm, int64_t b_sn) {
  return M > 0 && N > 0 && K > 0 && K % 8 == 0 && a_sm % 8 == 0 && b_sn % 8 == 0;
}

mla_status gemm_tc(const TcGemmArgs& g, cudaStream_t s) {
  if (g.M == 0 || g.N == 0) return MLA_OK;
  if (g.epilogue == kEpiRopeQ) {
    if (g.rope_D != 224 || g.N % 224 != 0)
      MLA_FAIL(MLA_ERR_UNSUPPORTED, "query RoPE epilogue needs 224-wide head blocks");
    return launch_gemm<224>(g, s);
  }
  // Tile width: the one whose CTA count fills whole waves of 148 SMs best (ties to the wider
  // tile, which re-reads A fewer times).  Projections here have few 128-row tiles, so a narrow
  // N tile is what puts every SM to work.
  constexpr int kSms = 148;
  const int widths[4] = {256, 224, 128, 64};
  int best = 256;
  double best_eff = -1.0;
  for (int w : widths) {
    const long long ctas =
        static_cast<long long>(ceil_div(g.M, kBM)) * ceil_div(g.N, w) * g.batch;
    const long long waves = (ctas + kSms - 1) / kSms;
    const double eff = static_cast<double>(ctas) / static_cast<double>(waves * kSms) *
                       (static_cast<double>(g.N) / (ceil_div(g.N, w) * w));
    if (eff > best_eff + 1e-9) {
      best_eff = eff;
      best = w;
    }
  }
  switch (best) {
    case 64: return launch_gemm<64>(g, s);
    case 128: return launch_gemm<128>(g, s);
    case 224: return launch_gemm<224>(g, s);
    default: return launch_gemm<256>(g, s);
  }
}

}  // namespace mla
