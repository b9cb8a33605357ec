// Stage (iii) of Lighthouse Attention: dense causal softmax attention over
// the gathered sub-sequence ("Long Context Pre-Training with Lighthouse
// Attention", Sec. 3.5, Eq. 9).  Because the gather is topologically sorted,
// the mask is the plain S x S causal one, so this is a causal attention
// forward on [BH, S, d] bf16 tensors, written for the sm_100a tensor cores.
//
// One CTA owns a tile of 128 query rows of one (b, h) and walks the key/value
// tiles of 128 rows up to the diagonal.  Warp roles:
//   warp 0     TMA producer: Q once, then K and V tiles into a 2-stage ring;
//   warp 1     tcgen05 issuer (one thread): S = Q K^T into one of two TMEM
//              score buffers, then O += P V into the TMEM accumulator; each
//              group is committed to an mbarrier;
//   warps 2-5  softmax, one query row per thread (TMEM lane = row): read the
//              score row from TMEM, online max / exp2 / row sum, write P as
//              bf16 into shared memory in the 128-byte-swizzled K-major layout
//              the next MMA reads, and rescale O in TMEM when the running
//              max of any row of the warp grew.
// The issuer computes S for tile j+1 while the softmax warps work on tile j
// and the tensor core runs P V for tile j-1.
//
// TMEM: two 128-column fp32 score buffers and a d-column fp32 accumulator
// (512 columns allocated, one CTA per SM).  Shared memory: Q (128 x d), two
// K and two V stages (128 x d each) and P (128 x 128), all bf16, 128-byte
// swizzled, 1024-byte aligned.
#include <cudaTypedefs.h>

#include "lh_sm100.cuh"

namespace {

using namespace sm100;

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int NST = 2;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;    // two score buffers: columns 0 and 128
constexpr uint32_t kColO = 256;  // accumulator

template <int HD>
struct FwdLayout {
  static constexpr uint32_t q = 0;
  static constexpr uint32_t k = q + BM * HD * 2;
  static constexpr uint32_t v = k + NST * BN * HD * 2;
  static constexpr uint32_t p = v + NST * BN * HD * 2;
  static constexpr uint32_t bar = p + BM * BN * 2;
  static constexpr uint32_t bytes = bar + 256;
};

// Force one CTA per SM (TMEM is allocated at 512 columns).
constexpr uint32_t kSmemBytes = FwdLayout<128>::bytes + 1024;

struct Bars {
  uint64_t qfull;
  uint64_t kfull[NST], kempty[NST], vfull[NST], vempty[NST];
  uint64_t sfull[2], sfree[2];
  uint64_t pfull, pvdone;
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
  uint8_t* pP = smem + Lay::p;
  const uint32_t sP = smem_u32(pP);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_qt = (S + BM - 1) / BM;
  const int qt = n_qt - 1 - (int)(blockIdx.x / BH);  // longest rows first
  const int bh = (int)(blockIdx.x % BH);
  const int n_kv = qt + 1;

  if (threadIdx.x == 0) {
    mbar_init(&bars->qfull, 1);
    for (int s = 0; s < NST; ++s) {
      mbar_init(&bars->kfull[s], 1);
      mbar_init(&bars->kempty[s], 1);
      mbar_init(&bars->vfull[s], 1);
      mbar_init(&bars->vempty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->sfull[s], 1);
      mbar_init(&bars->sfree[s], 128);
    }
    mbar_init(&bars->pfull, 128);
    mbar_init(&bars->pvdone, 1);
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
      mbar_expect_tx(&bars->qfull, BM * HD * 2);
      for (int blk = 0; blk < HD / 64; ++blk)
        tma_load_3d(&tmQ, &bars->qfull, smem + Lay::q + blk * BM * 128, 64 * blk, qt * BM, bh);
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
      auto pv = [&](int i) -> bool {
        const int s = i % NST;
        if (!mbar_wait(&bars->pfull, i & 1, status, 4)) return false;
        if (!mbar_wait(&bars->vfull[s], (i / NST) & 1, status, 5)) return false;
        tc_fence_after();
        const uint32_t vb = sV + s * BN * HD * 2;
#pragma unroll
        for (int ks = 0; ks < BN / 16; ++ks) {
          const uint64_t a = sdesc_sw128(sP + (ks >> 2) * BM * 128 + (ks & 3) * 32, 16, 1024);
          const uint64_t b = sdesc_sw128(vb + ks * 16 * 128, BN * 128, 1024);
          mma_bf16(tmem + kColO, a, b, idO, (i > 0 || ks > 0) ? 1u : 0u);
        }
        mma_commit(&bars->pvdone);
        mma_commit(&bars->vempty[s]);
        return true;
      };
      for (int j = 0; ok && j < n_kv; ++j) {
        const int s = j % NST;
        const int sb = j & 1;
        if (!mbar_wait(&bars->kfull[s], (j / NST) & 1, status, 6)) { ok = false; break; }
        if (!mbar_wait(&bars->sfree[sb], ((j >> 1) & 1) ^ 1, status, 7)) { ok = false; break; }
        tc_fence_after();
        const uint32_t kb = sK + s * BN * HD * 2;
#pragma unroll
        for (int ks = 0; ks < HD / 16; ++ks) {
          const uint64_t a = sdesc_sw128(sQ + (ks >> 2) * BM * 128 + (ks & 3) * 32, 16, 1024);
          const uint64_t b = sdesc_sw128(kb + (ks >> 2) * BN * 128 + (ks & 3) * 32, 16, 1024);
          mma_bf16(tmem + kColS + sb * BN, a, b, idS, ks > 0 ? 1u : 0u);
        }
        mma_commit(&bars->sfull[sb]);
        mma_commit(&bars->kempty[s]);
        if (j > 0 && !pv(j - 1)) { ok = false; break; }
      }
      if (ok) pv(n_kv - 1);
    }
  } else {
    // softmax warps: TMEM lane quarter = warp % 4
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;       // row in the tile
    const int qrow = qt * BM + r;            // row in the sequence
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    float m_used = -INFINITY, lsum = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const int sb = j & 1;
      if (!mbar_wait(&bars->sfull[sb], (j >> 1) & 1, status, 8)) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[BN / 32][32];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) tmem_ld32(tmem + lane_addr + kColS + sb * BN + c * 32, sr[c]);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&bars->sfree[sb]);
      const bool diag = (j == qt);
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < BN / 32; ++c)
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int col = c * 32 + e;
          const float x = __uint_as_float(sr[c][e]);
          if (!diag || col <= r) mx = fmaxf(mx, x);
        }
      // Exact running max: the row's largest term so far gets p = 1, which
      // bf16 holds exactly.  (Keeping a stale max, as a lazy-rescale scheme
      // does, rounds that dominant term by up to 2^-9 and the error reaches
      // D = rowsum(dO * O) of the backward unscaled.)
      const float m_new = fmaxf(m_used, mx * scale_log2);
      const bool grow = m_new > m_used;
      float alpha = 1.f;
      if (grow) {
        alpha = ex2(m_used - m_new);
        m_used = m_new;
      }
      float rs = 0.f;
      uint32_t pk[BN / 2];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c)
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const int col = c * 32 + e;
          float p0 = ex2(fmaf(__uint_as_float(sr[c][e]), scale_log2, -m_used));
          float p1 = ex2(fmaf(__uint_as_float(sr[c][e + 1]), scale_log2, -m_used));
          if (diag) {
            p0 = col <= r ? p0 : 0.f;
            p1 = col + 1 <= r ? p1 : 0.f;
          }
          rs += p0 + p1;
          pk[col >> 1] = pack_bf16x2(p0, p1);
        }
      lsum = lsum * alpha + rs;
      if (j > 0 && !mbar_wait(&bars->pvdone, (j - 1) & 1, status, 9)) { ok = false; break; }
      // P into the swizzled K-major layout: 16-byte chunk cc of row r at
      // block (col / 64), chunk (cc ^ (r % 8)).
#pragma unroll
      for (int q = 0; q < BN / 8; ++q) {
        const int blk = q >> 3, cc = q & 7;
        uint4 w;
        w.x = pk[q * 4 + 0]; w.y = pk[q * 4 + 1]; w.z = pk[q * 4 + 2]; w.w = pk[q * 4 + 3];
        *reinterpret_cast<uint4*>(pP + blk * BM * 128 + r * 128 + ((cc ^ (r & 7)) << 4)) = w;
      }
      if (j > 0 && __any_sync(0xffffffffu, grow)) {
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < HD / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_addr + kColO + c * 32, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(tmem + lane_addr + kColO + c * 32, o);
        }
        tmem_st_wait();
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(&bars->pfull);
    }
    if (ok && mbar_wait(&bars->pvdone, (n_kv - 1) & 1, status, 10)) {
      tc_fence_after();
      const float inv = 1.f / lsum;
#pragma unroll
      for (int c = 0; c < HD / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_addr + kColO + c * 32, o);
        tmem_ld_wait();
        if (qrow < S) {
          const int64_t base = ((int64_t)bh * S + qrow) * (HD / 8) + c * 4;
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            float x[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] = __uint_as_float(o[v * 8 + e]) * inv;
            uint4 w, r;
            w.x = pack_bf16x2(x[0], x[1]); w.y = pack_bf16x2(x[2], x[3]);
            w.z = pack_bf16x2(x[4], x[5]); w.w = pack_bf16x2(x[6], x[7]);
            og[base + v] = w;
            if (og_lo) {
              const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
              uint32_t rr[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 h = unpack_bf16x2(ww[e]);
                rr[e] = pack_bf16x2(x[2 * e] - h.x, x[2 * e + 1] - h.y);
              }
              r.x = rr[0]; r.y = rr[1]; r.z = rr[2]; r.w = rr[3];
              og_lo[base + v] = r;
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
  const dim3 grid((unsigned)(n_qt * BH));
  const float scale_log2 = scale * 1.4426950408889634f;
  if (d == 128) {
    static bool attr = false;
    if (!attr) {
      cudaFuncSetAttribute(k_attn_fwd<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
      attr = true;
    }
    k_attn_fwd<128><<<grid, kThreads, kSmemBytes, st>>>(tq, tk, tv, (uint4*)og, (uint4*)og_lo, lse,
                                                         (int)S, BH, scale_log2, status);
  } else if (d == 64) {
    static bool attr = false;
    if (!attr) {
      cudaFuncSetAttribute(k_attn_fwd<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
      attr = true;
    }
    k_attn_fwd<64><<<grid, kThreads, kSmemBytes, st>>>(tq, tk, tv, (uint4*)og, (uint4*)og_lo, lse,
                                                        (int)S, BH, scale_log2, status);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}
