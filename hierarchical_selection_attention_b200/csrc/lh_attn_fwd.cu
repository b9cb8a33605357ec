// Stage (iii) of Lighthouse Attention: dense causal softmax attention over
// the gathered sub-sequence ("Long Context Pre-Training with Lighthouse
// Attention", Sec. 3.5, Eq. 9).  Because the gather is topologically sorted,
// the mask is the plain S x S causal one, so this is a causal attention
// forward on [BH, S, d] bf16 tensors, written for the sm_100a tensor cores.
//
// One CTA owns two tiles of 128 query rows of one (b, h), A and B (rows
// 256 g .. 256 g + 255), and walks the key/value tiles of 128 rows up to B's
// diagonal (A skips the last one).  Warp roles:
//   warp 0      TMA producer: Q_A and Q_B once, then K and V tiles into a
//               2-stage ring;
//   warp 1      tcgen05 issuer (one thread).  Per key tile j it issues
//               S_A = Q_A K^T, S_B = Q_B K^T into TMEM, then, as each softmax
//               warpgroup hands back its P, O_X += P_X V with P_X read from
//               TMEM (A operand in tensor memory) and V from shared memory;
//   warps 2-5   softmax of tile A, warps 6-9 softmax of tile B: one query
//               row per thread (TMEM lane = row).  Each reads its score row,
//               keeps the exact running max and the row sum, writes
//               P = exp2(s - max) as bf16 pairs over the score columns it
//               has just read, and rescales O_X in TMEM when a row's max grew.
// While warpgroup A turns S_A into P_A, the tensor core works on S_B or on
// P_B V, and the other way round.
//
// TMEM (512 columns, one CTA per SM): S_A 0..127, S_B 128..255 (P_X packed
// into the first 64 columns of S_X), O_A and O_B (d columns each) from 256.
// Shared memory: Q_A, Q_B, two K and two V stages (128 x d bf16 each),
// 128-byte swizzled, 1024-byte aligned.
#include <cudaTypedefs.h>

#include "lh_sm100.cuh"

namespace {

using namespace sm100;

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int NST = 2;
constexpr int kThreads = 320;
constexpr uint32_t kTmemCols = 512;

template <int HD>
struct FwdLayout {
  static constexpr uint32_t q = 0;                       // Q_A, Q_B
  static constexpr uint32_t k = q + 2 * BM * HD * 2;
  static constexpr uint32_t v = k + NST * BN * HD * 2;
  static constexpr uint32_t bar = v + NST * BN * HD * 2;
  static constexpr uint32_t bytes = bar + 256;
};

// At least half the shared memory of an SM: one CTA per SM, since each
// allocates all 512 TMEM columns.
constexpr uint32_t kSmemBytes = FwdLayout<128>::bytes + 1024;
static_assert(kSmemBytes > 232448 / 2 && kSmemBytes <= 232448, "one CTA per SM");

struct Bars {
  uint64_t qfull;
  uint64_t kfull[NST], kempty[NST], vfull[NST], vempty[NST];
  uint64_t sfull[2], pfull[2], odone[2];
  uint32_t tmem_base;
};

template <int HD>
__global__ void __launch_bounds__(kThreads, 1)
    k_attn_fwd(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, uint4* __restrict__ og,
               uint4* __restrict__ og_lo, float* __restrict__ lse, int S, int BH,
               float scale_log2, int* status) {
  using Lay = FwdLayout<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  Bars* bars = reinterpret_cast<Bars*>(smem + Lay::bar);
  const uint32_t sQ = smem_u32(smem + Lay::q);
  const uint32_t sK = smem_u32(smem + Lay::k);
  const uint32_t sV = smem_u32(smem + Lay::v);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_qt = (S + BM - 1) / BM;
  const int n_pair = (n_qt + 1) / 2;
  const int g = n_pair - 1 - (int)(blockIdx.x / BH);  // longest rows first
  const int bh = (int)(blockIdx.x % BH);
  const int qt_a = 2 * g, qt_b = 2 * g + 1;
  const int n_a = qt_a + 1;                           // key tiles of tile A
  const int n_b = qt_b < n_qt ? qt_b + 1 : 0;         // 0: tile B is past the end
  const int n_kv = n_b ? n_b : n_a;

  if (threadIdx.x == 0) {
    mbar_init(&bars->qfull, 1);
    for (int s = 0; s < NST; ++s) {
      mbar_init(&bars->kfull[s], 1);
      mbar_init(&bars->kempty[s], 1);
      mbar_init(&bars->vfull[s], 1);
      mbar_init(&bars->vempty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bars->sfull[x], 1);
      mbar_init(&bars->pfull[x], 128);
      mbar_init(&bars->odone[x], 1);
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_expect_tx(&bars->qfull, 2 * BM * HD * 2);
      for (int x = 0; x < 2; ++x)
        for (int blk = 0; blk < HD / 64; ++blk)
          tma_load_3d(&tmQ, &bars->qfull, smem + Lay::q + x * BM * HD * 2 + blk * BM * 128,
                      64 * blk, (qt_a + x) * BM, bh);
      for (int j = 0; j < n_kv; ++j) {
        const int s = j % NST;
        const uint32_t ph = (j / NST) & 1;
        if (!mbar_wait(&bars->kempty[s], ph ^ 1, status, 1)) break;
        mbar_expect_tx(&bars->kfull[s], BN * HD * 2);
        for (int blk = 0; blk < HD / 64; ++blk)
          tma_load_3d(&tmK, &bars->kfull[s], smem + Lay::k + s * BN * HD * 2 + blk * BN * 128,
                      64 * blk, j * BN, bh);
        if (!mbar_wait(&bars->vempty[s], ph ^ 1, status, 2)) break;
        mbar_expect_tx(&bars->vfull[s], BN * HD * 2);
        for (int blk = 0; blk < HD / 64; ++blk)
          tma_load_3d(&tmV, &bars->vfull[s], smem + Lay::v + s * BN * HD * 2 + blk * BN * 128,
                      64 * blk, j * BN, bh);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(BM, BN, 0, 0);
      constexpr uint32_t idO = idesc_bf16(BM, HD, 0, 1);
      bool ok = mbar_wait(&bars->qfull, 0, status, 3);
      for (int j = 0; ok && j < n_kv; ++j) {
        const int s = j % NST;
        const uint32_t ph = (j / NST) & 1;
        if (!mbar_wait(&bars->kfull[s], ph, status, 4)) { ok = false; break; }
        const uint32_t kb = sK + s * BN * HD * 2;
        for (int x = 0; x < 2 && ok; ++x) {
          if (j >= (x ? n_b : n_a)) continue;
          // S_X shares its columns with P_X of the last tile: P_X V must be done
          if (j > 0 && !mbar_wait(&bars->odone[x], (j - 1) & 1, status, 5)) { ok = false; break; }
          tc_fence_after();
          const uint32_t qb = sQ + x * BM * HD * 2;
#pragma unroll
          for (int ks = 0; ks < HD / 16; ++ks) {
            const uint64_t a = sdesc_sw128(qb + (ks >> 2) * BM * 128 + (ks & 3) * 32, 16, 1024);
            const uint64_t b = sdesc_sw128(kb + (ks >> 2) * BN * 128 + (ks & 3) * 32, 16, 1024);
            mma_bf16(tmem + x * 128, a, b, idS, ks > 0 ? 1u : 0u);
          }
          mma_commit(&bars->sfull[x]);
        }
        if (!ok) break;
        mma_commit(&bars->kempty[s]);
        if (!mbar_wait(&bars->vfull[s], ph, status, 6)) { ok = false; break; }
        const uint32_t vb = sV + s * BN * HD * 2;
        for (int x = 0; x < 2 && ok; ++x) {
          if (j >= (x ? n_b : n_a)) continue;
          if (!mbar_wait(&bars->pfull[x], j & 1, status, 7)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < BN / 16; ++ks) {
            const uint64_t b = sdesc_sw128(vb + ks * 16 * 128, BN * 128, 1024);
            mma_bf16_ts(tmem + 256 + x * HD, tmem + x * 128 + ks * 8, b, idO,
                        (j > 0 || ks > 0) ? 1u : 0u);
          }
          mma_commit(&bars->odone[x]);
        }
        if (!ok) break;
        mma_commit(&bars->vempty[s]);
      }
    }
  } else {
    // softmax warpgroup x: warps 2-5 (x = 0) and 6-9 (x = 1)
    const int x = (warp - 2) >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;       // row in the tile = TMEM lane
    const int qt = qt_a + x;
    const int qrow = qt * BM + r;            // row in the sequence
    const int n_x = x ? n_b : n_a;
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_addr + x * 128;
    const uint32_t tO = tmem + lane_addr + 256 + x * HD;
    float m_used = -INFINITY, lsum = 0.f;
    bool ok = true;
    for (int j = 0; j < n_x; ++j) {
      if (!mbar_wait(&bars->sfull[x], j & 1, status, 8)) { ok = false; break; }
      tc_fence_after();
      // Two passes over the score row in TMEM, two 32-column chunks at a
      // time: the max first, then exp2 / sum / pack.  Holding the whole row
      // in registers would spill at this block size.
      const bool diag = (j == qt);
      float mxv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) mxv[u] = -INFINITY;
#pragma unroll
      for (int c = 0; c < BN / 32; c += 2) {
        uint32_t a[32], b[32];
        tmem_ld32(tS + c * 32, a);
        tmem_ld32(tS + c * 32 + 32, b);
        tmem_ld_wait();
        if (diag) {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            if (c * 32 + e <= r) mxv[e & 7] = fmaxf(mxv[e & 7], __uint_as_float(a[e]));
            if (c * 32 + 32 + e <= r) mxv[e & 7] = fmaxf(mxv[e & 7], __uint_as_float(b[e]));
          }
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e)
            mxv[e & 7] = fmaxf(mxv[e & 7], fmaxf(__uint_as_float(a[e]), __uint_as_float(b[e])));
        }
      }
      const float mx = fmaxf(fmaxf(fmaxf(mxv[0], mxv[1]), fmaxf(mxv[2], mxv[3])),
                             fmaxf(fmaxf(mxv[4], mxv[5]), fmaxf(mxv[6], mxv[7])));
      // Exact running max: the row's largest term so far gets p = 1, which
      // bf16 holds exactly.  (A stale max, as lazy rescaling keeps, would
      // round that dominant term by up to 2^-9, and the error would reach
      // D = rowsum(dO * O) of the backward unscaled.)
      const float m_new = fmaxf(m_used, mx * scale_log2);
      const bool grow = m_new > m_used;
      const float alpha = grow ? ex2(m_used - m_new) : 1.f;
      m_used = m_new;
      float rsv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) rsv[u] = 0.f;
#pragma unroll
      for (int c = 0; c < BN / 32; c += 2) {
        uint32_t a[32], b[32];
        tmem_ld32(tS + c * 32, a);
        tmem_ld32(tS + c * 32 + 32, b);
        tmem_ld_wait();
        uint32_t pa[16], pb[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float p0 = ex2(fmaf(__uint_as_float(a[e]), scale_log2, -m_used));
          float p1 = ex2(fmaf(__uint_as_float(a[e + 1]), scale_log2, -m_used));
          float q0 = ex2(fmaf(__uint_as_float(b[e]), scale_log2, -m_used));
          float q1 = ex2(fmaf(__uint_as_float(b[e + 1]), scale_log2, -m_used));
          if (diag) {
            p0 = (c * 32 + e <= r) ? p0 : 0.f;
            p1 = (c * 32 + e + 1 <= r) ? p1 : 0.f;
            q0 = (c * 32 + 32 + e <= r) ? q0 : 0.f;
            q1 = (c * 32 + 32 + e + 1 <= r) ? q1 : 0.f;
          }
          rsv[(e >> 1) & 7] += (p0 + p1) + (q0 + q1);
          pa[e >> 1] = pack_bf16x2(p0, p1);
          pb[e >> 1] = pack_bf16x2(q0, q1);
        }
        // P over columns of this row already read (pair c covers 64 score
        // columns from c * 32 and packs into 32 columns from c * 16)
        tmem_st16(tS + c * 16, pa);
        tmem_st16(tS + c * 16 + 16, pb);
      }
      const float rs = ((rsv[0] + rsv[1]) + (rsv[2] + rsv[3])) + ((rsv[4] + rsv[5]) + (rsv[6] + rsv[7]));
      lsum = lsum * alpha + rs;
      // O_X holds P V of the earlier tiles (P_X V of tile j-1 finished before
      // S_X of tile j was issued); bring it to the new max.
      if (j > 0 && __any_sync(0xffffffffu, grow)) {
#pragma unroll
        for (int c = 0; c < HD / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + c * 32, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(tO + c * 32, o);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars->pfull[x]);
    }
    if (ok && n_x > 0 && mbar_wait(&bars->odone[x], (n_x - 1) & 1, status, 10)) {
      tc_fence_after();
      const float inv = 1.f / lsum;
#pragma unroll
      for (int c = 0; c < HD / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + c * 32, o);
        tmem_ld_wait();
        if (qrow < S) {
          const int64_t base = ((int64_t)bh * S + qrow) * (HD / 8) + c * 4;
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            float xv[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) xv[e] = __uint_as_float(o[v * 8 + e]) * inv;
            uint4 w;
            w.x = pack_bf16x2(xv[0], xv[1]); w.y = pack_bf16x2(xv[2], xv[3]);
            w.z = pack_bf16x2(xv[4], xv[5]); w.w = pack_bf16x2(xv[6], xv[7]);
            og[base + v] = w;
            if (og_lo) {
              const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
              uint32_t rr[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 hh = unpack_bf16x2(ww[e]);
                rr[e] = pack_bf16x2(xv[2 * e] - hh.x, xv[2 * e + 1] - hh.y);
              }
              og_lo[base + v] = make_uint4(rr[0], rr[1], rr[2], rr[3]);
            }
          }
        }
      }
      if (qrow < S) lse[(int64_t)bh * S + qrow] = (m_used + __log2f(lsum)) * 0.69314718055994531f;
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

}  // namespace

// Tensor map over a [BH, rows, d] bf16 tensor, box = 64 features x box_rows
// rows of one (b, h), 128-byte swizzle; rows past `rows` read as zero.
bool lh_make_tmap_3d(CUtensorMap* m, const void* base, int64_t BH, int64_t rows, int d,
                     int box_rows) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)rows, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)rows * d * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

cudaError_t lh_launch_attn_fwd(int BH, int64_t S, int d, float scale, const lh_bf16* qg,
                               const lh_bf16* kg, const lh_bf16* vg, lh_bf16* og,
                               lh_bf16* og_lo, float* lse, int* status, cudaStream_t st) {
  CUtensorMap tq, tk, tv;
  if (!lh_make_tmap_3d(&tq, qg, BH, S, d, BM) || !lh_make_tmap_3d(&tk, kg, BH, S, d, BN) ||
      !lh_make_tmap_3d(&tv, vg, BH, S, d, BN))
    return cudaErrorInvalidValue;
  const int n_qt = (int)((S + BM - 1) / BM);
  const dim3 grid((unsigned)(((n_qt + 1) / 2) * BH));
  const float scale_log2 = scale * 1.4426950408889634f;
  if (d == 128) {
    cudaFuncSetAttribute(k_attn_fwd<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    k_attn_fwd<128><<<grid, kThreads, kSmemBytes, st>>>(tq, tk, tv, (uint4*)og, (uint4*)og_lo, lse,
                                                         (int)S, BH, scale_log2, status);
  } else if (d == 64) {
    cudaFuncSetAttribute(k_attn_fwd<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    k_attn_fwd<64><<<grid, kThreads, kSmemBytes, st>>>(tq, tk, tv, (uint4*)og, (uint4*)og_lo, lse,
                                                        (int)S, BH, scale_log2, status);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}
