// Plain bf16 GEMMs for the projections on either side of the layer: per-head
// Q, K, V come from the layer's own W_Q, W_K, W_V, and an output projection
// follows ("Long Context Pre-Training with Lighthouse Attention", Sec. 3.1).
// Their backward needs the same products with transposed operands and the
// weight gradients, so one kernel covers
//      C[M, N] = sum_i A_i[M, K_i] B_i[N, K_i]^T      (i < 3, fp32 accumulate)
// with A and B each stored K-major (K contiguous) or MN-major (M or N
// contiguous), and an optional split of the K range over CTAs whose fp32
// partials a second kernel sums in a fixed order (deterministic).
//
// sm_100a design: a persistent kernel, one CTA per SM, 128 x 256 output
// tiles.  Warp 0 streams 128 x 64 slices of A and 256 x 64 slices of B with
// TMA (128-byte swizzle) into a 4-stage ring; warp 1 issues tcgen05 MMAs
// (whole-warp loop, one lane issues) into one of two TMEM accumulators
// (256 columns each); warps 2-5 read the other accumulator back, round it
// and store it, so a tile's epilogue overlaps the next tile's MMAs.
#include <cudaTypedefs.h>

#include <cstring>

#include "lh_sm100.cuh"

PFN_cuTensorMapEncodeTiled_v12000 lh_tensormap_encoder();

namespace {

using namespace sm100;

constexpr int GM = 128, GN = 256, GK = 64, GST = 4;
constexpr int kGemmThreads = 192;
constexpr int kMaxPairs = 3;
constexpr uint32_t kStageA = GM * GK * 2;          // 16 KB
constexpr uint32_t kStageB = GN * GK * 2;          // 32 KB
constexpr uint32_t kSmemGemm = GST * (kStageA + kStageB) + 256 + 1024;
static_assert(kSmemGemm <= 232448 && kSmemGemm > 232448 / 2, "one CTA per SM");

struct GemmBars {
  uint64_t full[GST], empty[GST], accfull[2], accempty[2];
  uint32_t tmem_base;
};

struct GemmMaps {
  CUtensorMap a[kMaxPairs], b[kMaxPairs];
};

struct GemmShape {
  int M, N, npairs, splits;
  int ksteps[kMaxPairs];   // 64-wide K slices of each pair
  int total;               // sum of ksteps
  int tiles_n, units;      // units = tiles * splits
  int64_t ldc;
  int f32_out;             // 1: fp32 partials [splits][M][N]; 0: bf16 C
  int* status;
};

__device__ __forceinline__ void tma_load_2d(const CUtensorMap* m, uint64_t* bar, void* dst, int c0,
                                            int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}

// Unit u -> output tile (tm, tn) and K split; the n tiles of one m row are
// neighbours so concurrent CTAs share A rows in L2.
__device__ __forceinline__ void unit_of(const GemmShape& G, int u, int& tm, int& tn, int& s0,
                                        int& s1) {
  const int sp = u % G.splits, t = u / G.splits;
  tm = t / G.tiles_n;
  tn = t % G.tiles_n;
  const int per = (G.total + G.splits - 1) / G.splits;
  s0 = sp * per;
  s1 = min(G.total, s0 + per);
}

template <bool A_MN, bool B_MN>
__global__ void __launch_bounds__(kGemmThreads, 1)
    k_gemm(const __grid_constant__ GemmMaps maps, const GemmShape G, void* __restrict__ c) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  uint8_t* sA = smem;
  uint8_t* sB = smem + GST * kStageA;
  GemmBars* bars = reinterpret_cast<GemmBars*>(smem + GST * (kStageA + kStageB));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < GST; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->accfull[b], 1);
      mbar_init(&bars->accempty[b], 128);
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      int it = 0;                                      // ring position across units
      bool ok = true;
      for (int u = blockIdx.x; ok && u < G.units; u += gridDim.x) {
        int tm, tn, s0, s1;
        unit_of(G, u, tm, tn, s0, s1);
        // walk the pairs to the first slice of this unit
        int pair = 0, base = 0;
        while (pair + 1 < G.npairs && s0 >= base + G.ksteps[pair]) base += G.ksteps[pair++];
        for (int g = s0; g < s1; ++g, ++it) {
          while (g >= base + G.ksteps[pair]) base += G.ksteps[pair++];
          const int s = it % GST;
          if (!mbar_wait(&bars->empty[s], ((it / GST) & 1) ^ 1, G.status, 60)) { ok = false; break; }
          mbar_expect_tx(&bars->full[s], kStageA + kStageB);
          const int k0 = (g - base) * GK, m0 = tm * GM, n0 = tn * GN;
          if (A_MN) {
            for (int blk = 0; blk < GM / 64; ++blk)
              tma_load_2d(&maps.a[pair], &bars->full[s], sA + s * kStageA + blk * 64 * GK * 2,
                          m0 + 64 * blk, k0);
          } else {
            tma_load_2d(&maps.a[pair], &bars->full[s], sA + s * kStageA, k0, m0);
          }
          if (B_MN) {
            for (int blk = 0; blk < GN / 64; ++blk)
              tma_load_2d(&maps.b[pair], &bars->full[s], sB + s * kStageB + blk * 64 * GK * 2,
                          n0 + 64 * blk, k0);
          } else {
            tma_load_2d(&maps.b[pair], &bars->full[s], sB + s * kStageB, k0, n0);
          }
        }
      }
    }
  } else if (warp == 1) {
    constexpr uint32_t id = idesc_bf16(GM, GN, A_MN ? 1 : 0, B_MN ? 1 : 0);
    const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
    int it = 0, n_unit = 0;
    bool ok = true;
    for (int u = blockIdx.x; ok && u < G.units; u += gridDim.x, ++n_unit) {
      int tm, tn, s0, s1;
      unit_of(G, u, tm, tn, s0, s1);
      const int b = n_unit & 1;
      if (!mbar_wait_w(&bars->accempty[b], ((n_unit >> 1) & 1) ^ 1, G.status, 61)) break;
      tc_fence_after();
      for (int g = s0; g < s1; ++g, ++it) {
        const int s = it % GST;
        if (!mbar_wait_w(&bars->full[s], (it / GST) & 1, G.status, 62)) { ok = false; break; }
        tc_fence_after();
        const uint32_t as = a0 + s * kStageA, bs = b0 + s * kStageB;
#pragma unroll
        for (int ks = 0; ks < GK / 16; ++ks) {
          const uint64_t ad = A_MN ? sdesc_sw128(as + ks * 16 * 128, 64 * GK * 2, 1024)
                                   : sdesc_sw128(as + ks * 32, 16, 1024);
          const uint64_t bd = B_MN ? sdesc_sw128(bs + ks * 16 * 128, 64 * GK * 2, 1024)
                                   : sdesc_sw128(bs + ks * 32, 16, 1024);
          mma_bf16_w(tmem + b * GN, ad, bd, id, (g > s0 || ks > 0) ? 1u : 0u);
        }
        mma_commit_w(&bars->empty[s]);
      }
      if (!ok) break;
      mma_commit_w(&bars->accfull[b]);
    }
  } else {
    // epilogue: warps 2-5, TMEM lane quarter = warp % 4, one output row each
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    int n_unit = 0;
    for (int u = blockIdx.x; u < G.units; u += gridDim.x, ++n_unit) {
      int tm, tn, s0, s1;
      unit_of(G, u, tm, tn, s0, s1);
      const int b = n_unit & 1;
      if (!mbar_wait_w(&bars->accfull[b], (n_unit >> 1) & 1, G.status, 63)) break;
      tc_fence_after();
      const int m = tm * GM + r;
      const int sp = u % G.splits;
#pragma unroll 1
      for (int cc = 0; cc < GN / 32; ++cc) {
        uint32_t x[32];
        tmem_ld32(tmem + lane_addr + b * GN + cc * 32, x);
        tmem_ld_wait();
        const int n = tn * GN + cc * 32;
        if (m >= G.M || n >= G.N) continue;
        if (G.f32_out) {
          float* row = reinterpret_cast<float*>(c) + ((int64_t)sp * G.M + m) * G.N;
#pragma unroll
          for (int v = 0; v < 8; ++v)
            if (n + 4 * v < G.N)
              *reinterpret_cast<float4*>(row + n + 4 * v) =
                  make_float4(__uint_as_float(x[4 * v]), __uint_as_float(x[4 * v + 1]),
                              __uint_as_float(x[4 * v + 2]), __uint_as_float(x[4 * v + 3]));
        } else {
          uint4* row = reinterpret_cast<uint4*>(reinterpret_cast<lh_bf16*>(c) + m * G.ldc + n);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            if (n + 8 * v < G.N)
              row[v] = make_uint4(pack_bf16x2(__uint_as_float(x[8 * v]), __uint_as_float(x[8 * v + 1])),
                                  pack_bf16x2(__uint_as_float(x[8 * v + 2]), __uint_as_float(x[8 * v + 3])),
                                  pack_bf16x2(__uint_as_float(x[8 * v + 4]), __uint_as_float(x[8 * v + 5])),
                                  pack_bf16x2(__uint_as_float(x[8 * v + 6]), __uint_as_float(x[8 * v + 7])));
        }
      }
      tc_fence_before();
      mbar_arrive(&bars->accempty[b]);
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// C[m, n] = bf16(sum over splits of the fp32 partials), splits in order.
__global__ void __launch_bounds__(256) k_gemm_reduce(const float* __restrict__ part, int M, int N,
                                                     int splits, lh_bf16* __restrict__ c,
                                                     int64_t ldc) {
  const int64_t groups = (int64_t)M * (N / 8);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < groups;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t m = i / (N / 8);
    const int n = (int)(i - m * (N / 8)) * 8;
    float a[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int s = 0; s < splits; ++s) {
      const float4* p = reinterpret_cast<const float4*>(part + ((int64_t)s * M + m) * N + n);
      const float4 x = __ldg(p), y = __ldg(p + 1);
      a[0] += x.x; a[1] += x.y; a[2] += x.z; a[3] += x.w;
      a[4] += y.x; a[5] += y.y; a[6] += y.z; a[7] += y.w;
    }
    *reinterpret_cast<uint4*>(c + m * ldc + n) =
        make_uint4(pack_bf16x2(a[0], a[1]), pack_bf16x2(a[2], a[3]), pack_bf16x2(a[4], a[5]),
                   pack_bf16x2(a[6], a[7]));
  }
}

bool make_map_2d(CUtensorMap* m, const void* base, int64_t inner, int64_t outer, int64_t ld,
                 int box_inner, int box_outer) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = lh_tensormap_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {(cuuint32_t)box_inner, (cuuint32_t)box_outer};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool A_MN, bool B_MN>
cudaError_t launch(const GemmMaps& maps, const GemmShape& G, void* c, int grid, cudaStream_t st) {
  cudaFuncSetAttribute(k_gemm<A_MN, B_MN>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemGemm);
  k_gemm<A_MN, B_MN><<<grid, kGemmThreads, kSmemGemm, st>>>(maps, G, c);
  return cudaGetLastError();
}

}  // namespace

size_t lh_gemm_partial_bytes(int64_t M, int64_t N, int splits) {
  return splits > 1 ? (size_t)splits * M * N * sizeof(float) : 0;
}

cudaError_t lh_launch_gemm(int64_t M, int64_t N, int npairs, const lh_gemm_operand* ops, int a_mn,
                           int b_mn, lh_bf16* c, int64_t ldc, int splits, void* ws, int* status,
                           int num_sms, cudaStream_t st, int* launches) {
  GemmMaps maps;
  GemmShape G;
  memset(&maps, 0, sizeof(maps));
  memset(&G, 0, sizeof(G));
  G.M = (int)M;
  G.N = (int)N;
  G.npairs = npairs;
  G.splits = splits;
  for (int i = 0; i < npairs; ++i) {
    const lh_gemm_operand& o = ops[i];
    G.ksteps[i] = (int)((o.k + GK - 1) / GK);
    G.total += G.ksteps[i];
    const bool okA = a_mn ? make_map_2d(&maps.a[i], o.a, M, o.k, o.lda, 64, 64)
                          : make_map_2d(&maps.a[i], o.a, o.k, M, o.lda, 64, GM);
    const bool okB = b_mn ? make_map_2d(&maps.b[i], o.b, N, o.k, o.ldb, 64, 64)
                          : make_map_2d(&maps.b[i], o.b, o.k, N, o.ldb, 64, GN);
    if (!okA || !okB) return cudaErrorInvalidValue;
  }
  // no empty split: with per = ceil(total / splits), ceil(total / per) splits
  const int per = (G.total + splits - 1) / splits;
  splits = (G.total + per - 1) / per;
  G.splits = splits;
  G.tiles_n = (int)((N + GN - 1) / GN);
  const int64_t tiles = ((M + GM - 1) / GM) * G.tiles_n;
  G.units = (int)(tiles * splits);
  G.ldc = ldc;
  G.f32_out = splits > 1;
  G.status = status;
  const int grid = G.units < num_sms ? G.units : num_sms;
  void* out = splits > 1 ? ws : (void*)c;
  cudaError_t e;
  if (!a_mn && !b_mn) e = launch<false, false>(maps, G, out, grid, st);
  else if (!a_mn && b_mn) e = launch<false, true>(maps, G, out, grid, st);
  else if (a_mn && !b_mn) e = launch<true, false>(maps, G, out, grid, st);
  else e = launch<true, true>(maps, G, out, grid, st);
  int n = 1;
  if (e == cudaSuccess && splits > 1) {
    const int64_t groups = M * (N / 8);
    const int blocks = (int)((groups + 255) / 256 < 148 * 8 ? (groups + 255) / 256 : 148 * 8);
    k_gemm_reduce<<<blocks, 256, 0, st>>>((const float*)ws, (int)M, (int)N, splits, c, ldc);
    e = cudaGetLastError();
    ++n;
  }
  if (launches) *launches = n;
  return e;
}
