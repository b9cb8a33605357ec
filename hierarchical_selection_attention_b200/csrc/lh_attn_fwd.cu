// Stage (iii) of Lighthouse Attention: dense causal softmax attention over
// the gathered sub-sequence ("Long Context Pre-Training with Lighthouse
// Attention", Sec. 3.5, Eq. 9).  Because the gather is topologically sorted,
// the mask is the plain S x S causal one, so this is a causal attention
// forward on [BH, S, d] bf16 tensors, written for the sm_100a tensor cores.
//
// One CTA owns one tile of 128 query rows of one (b, h) and walks the
// key/value tiles of 128 rows up to its diagonal.  Warp roles:
//   warp 0      TMA producer: Q once, then K and V tiles into their rings;
//   warp 1      issuer A: S(j) = Q K(j)^T into TMEM score buffer j % 2;
//   warp 10     issuer B: O_h += P_h(j) V_h(j) for the two column halves h
//               (keys 64 h .. 64 h + 63 of the tile), P_h read from TMEM (A
//               operand in tensor memory), V from shared memory;
//   warps 2-9   two softmax warpgroups; warpgroup h owns columns 64 h ..
//               64 h + 63 of every score row, one row per thread (TMEM lane
//               = row), with its own exact running max, row sum and output
//               accumulator O_h: a split of the key dimension in two inside
//               the CTA, so the warpgroups never exchange anything per tile.
//               The epilogue merges the halves: with m = max(m_0, m_1),
//               O = (O_0 2^(m_0 - m) + O_1 2^(m_1 - m)) / (l_0 2^(m_0 - m) +
//               l_1 2^(m_1 - m)).
// With two score buffers S(j + 1) is computed while the softmax works on
// S(j), and P(j) V(j) runs while it works on S(j + 1), so the tensor pipe and
// the softmax overlap.  The issuers run whole-warp loops (one lane issues).
//
// TMEM (512 columns, one CTA per SM): score buffers 0..127 and 128..255
// (P_h packed into the first 32 columns of its half), O_0 from 256 and O_1
// from 256 + d.  Shared memory: Q, KST K stages and VST V stages (128 x d
// bf16 each), 128-byte swizzled, 1024-byte aligned, and the merge buffer.
//
// Blocks of a ring (context parallelism, the pages' multi-GPU training
// note: the gathered sub-sequences of consecutive shards rotate through
// ring attention).  The same kernel computes one step of it: the rows of
// one shard's sub-sequence against one K/V block of the same length S,
// either the shard's own block (causal, as above) or an earlier shard's
// block (`full`: every key visible; keys past S masked).  Partial results
// merge by log-sum-exp into fp32 accumulators, in base 2:
//   lse2 = log2(2^a + 2^b),  O = O_a 2^(a - lse2) + O_b 2^(b - lse2)
// with a the accumulated and b this block's lse2 and O_a, O_b normalised.
// `first` writes the accumulators without reading them; `last` writes the
// bf16 output and natural-log LSE instead of them.  first && last is the
// plain single-block attention.
#include <cudaTypedefs.h>

#include <type_traits>

#include "lh_sm100.cuh"

namespace {

using namespace sm100;

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int KST = 3;
constexpr int VST = 2;
constexpr int kThreads = 352;
constexpr int kHalf = 128;           // threads of one softmax warpgroup
constexpr uint32_t kTmemCols = 512;

template <int HD>
struct FwdLayout {
  static constexpr uint32_t q = 0;
  static constexpr uint32_t k = q + BM * HD * 2;
  static constexpr uint32_t v = k + KST * BN * HD * 2;
  static constexpr uint32_t merge = v + VST * BN * HD * 2;   // [2][128] (m, l) pairs
  static constexpr uint32_t bar = merge + 2 * BM * 8;
  static constexpr uint32_t bytes = bar + 256;
};

// At least half the shared memory of an SM: one CTA per SM, since each
// allocates all 512 TMEM columns.
constexpr uint32_t kSmemBytes = FwdLayout<128>::bytes + 1024;
static_assert(kSmemBytes > 232448 / 2 && kSmemBytes <= 232448, "one CTA per SM");

struct Bars {
  // Indexed by score buffer (tile parity), so a fast side can never
  // complete a barrier twice before the other side has seen the first phase.
  uint64_t qfull;
  uint64_t kfull[KST], kempty[KST], vfull[VST], vempty[VST];
  uint64_t sfull[2], pfull[2][2], pvdone[2];
  uint32_t tmem_base;
};

template <int HD>
__global__ void __launch_bounds__(kThreads, 1)
    k_attn_fwd(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, uint4* __restrict__ og,
               uint4* __restrict__ og_lo, float* __restrict__ lse, int S, int BH,
               float scale_log2, int* status, int full, int first, int last,
               float* __restrict__ o_acc, float* __restrict__ lse2_acc) {
  using Lay = FwdLayout<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  Bars* bars = reinterpret_cast<Bars*>(smem + Lay::bar);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_qt = (S + BM - 1) / BM;
  const int qt = n_qt - 1 - (int)(blockIdx.x / BH);  // longest rows first
  const int bh = (int)(blockIdx.x % BH);
  // key tiles up to the diagonal (BN == BM), or all of them for an earlier block
  const int n_kv = full ? n_qt : qt + 1;

  if (threadIdx.x == 0) {
    mbar_init(&bars->qfull, 1);
    for (int s = 0; s < KST; ++s) {
      mbar_init(&bars->kfull[s], 1);
      mbar_init(&bars->kempty[s], 1);
    }
    for (int s = 0; s < VST; ++s) {
      mbar_init(&bars->vfull[s], 1);
      mbar_init(&bars->vempty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->sfull[b], 1);
      mbar_init(&bars->pfull[b][0], kHalf);
      mbar_init(&bars->pfull[b][1], kHalf);
      mbar_init(&bars->pvdone[b], 1);
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
      mbar_expect_tx(&bars->qfull, BM * HD * 2);
      for (int blk = 0; blk < HD / 64; ++blk)
        tma_load_3d(&tmQ, &bars->qfull, smem + Lay::q + blk * BM * 128, 64 * blk, qt * BM, bh);
      for (int j = 0; j < n_kv; ++j) {
        const int s = j % KST, t = j % VST;
        if (!mbar_wait(&bars->kempty[s], ((j / KST) & 1) ^ 1, status, 1)) break;
        mbar_expect_tx(&bars->kfull[s], BN * HD * 2);
        for (int blk = 0; blk < HD / 64; ++blk)
          tma_load_3d(&tmK, &bars->kfull[s], smem + Lay::k + s * BN * HD * 2 + blk * BN * 128,
                      64 * blk, j * BN, bh);
        if (!mbar_wait(&bars->vempty[t], ((j / VST) & 1) ^ 1, status, 2)) break;
        mbar_expect_tx(&bars->vfull[t], BN * HD * 2);
        for (int blk = 0; blk < HD / 64; ++blk)
          tma_load_3d(&tmV, &bars->vfull[t], smem + Lay::v + t * BN * HD * 2 + blk * BN * 128,
                      64 * blk, j * BN, bh);
      }
    }
  } else if (warp == 1) {
    // Issuer A: S(j) = Q K(j)^T into buffer j % 2, once P(j - 2) V(j - 2)
    // (which read P(j - 2) from that buffer) has finished.
    constexpr uint32_t idS = idesc_bf16(BM, BN, 0, 0);
    const uint32_t sQ = smem_u32(smem + Lay::q), sK = smem_u32(smem + Lay::k);
    bool ok = mbar_wait_w(&bars->qfull, 0, status, 3);
    for (int j = 0; ok && j < n_kv; ++j) {
      const int s = j % KST, b = j & 1;
      if (!mbar_wait_w(&bars->kfull[s], (j / KST) & 1, status, 4)) break;
      if (j >= 2 && !mbar_wait_w(&bars->pvdone[b], ((j >> 1) & 1) ^ 1, status, 5)) break;
      tc_fence_after();
      const uint32_t kb = sK + s * BN * HD * 2;
#pragma unroll
      for (int ks = 0; ks < HD / 16; ++ks) {
        const uint64_t a = sdesc_sw128(sQ + (ks >> 2) * BM * 128 + (ks & 3) * 32, 16, 1024);
        const uint64_t bd = sdesc_sw128(kb + (ks >> 2) * BN * 128 + (ks & 3) * 32, 16, 1024);
        mma_bf16_w(tmem + b * BN, a, bd, idS, ks > 0 ? 1u : 0u);
      }
      mma_commit_w(&bars->sfull[b]);
      mma_commit_w(&bars->kempty[s]);
    }
  } else if (warp == 10) {
    // Issuer B: O_h += P_h(j) V_h(j) as each softmax warpgroup hands back its
    // half of P(j) (and has rescaled O_h for tile j's max).
    constexpr uint32_t idO = idesc_bf16(BM, HD, 0, 1);
    const uint32_t sV = smem_u32(smem + Lay::v);
    bool ok = true;
    for (int j = 0; ok && j < n_kv; ++j) {
      const int t = j % VST, b = j & 1;
      if (!mbar_wait_w(&bars->vfull[t], (j / VST) & 1, status, 6)) break;
      const uint32_t vb = sV + t * BN * HD * 2;
      for (int h = 0; h < 2; ++h) {
        if (!mbar_wait_w(&bars->pfull[b][h], (j >> 1) & 1, status, 7)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < BN / 32; ++ks)
          mma_bf16_ts_w(tmem + 256 + h * HD, tmem + b * BN + h * 64 + ks * 8,
                        sdesc_sw128(vb + (h * 4 + ks) * 16 * 128, BN * 128, 1024), idO,
                        (j > 0 || ks > 0) ? 1u : 0u);
      }
      if (!ok) break;
      mma_commit_w(&bars->pvdone[b]);
      mma_commit_w(&bars->vempty[t]);
    }
  } else {
    // softmax warpgroup h (warps 2-5: h = 0, 6-9: h = 1); TMEM lane quarter =
    // warp % 4.  Waits are warp-wide (the vote below needs every lane).
    const int h = (warp - 2) >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;       // row in the tile = TMEM lane
    const int qrow = qt * BM + r;            // row in the sequence
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    const uint32_t tO = tmem + lane_addr + 256 + h * HD;
    const int c0 = h * 64;                   // first column of this half
    float m_used = -INFINITY, lsum = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const int b = j & 1;
      const uint32_t tS = tmem + lane_addr + b * BN + c0;
      if (!mbar_wait_w(&bars->sfull[b], (j >> 1) & 1, status, 8)) { ok = false; break; }
      tc_fence_after();
      uint32_t s[64];
      tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
      tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
      tmem_ld_wait();
      // masked tile: the diagonal (keys <= r) or, for an earlier block, the
      // ragged last tile (keys < S); columns c0 + e < lim are kept
      const bool diag = !full && (j == qt);
      const bool msk = diag || (full && (j + 1) * BN > S);
      const int lim = diag ? r + 1 : S - j * BN;
      float mxv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) mxv[u] = -INFINITY;
      if (msk) {
#pragma unroll
        for (int e = 0; e < 64; ++e)
          if (c0 + e < lim) mxv[e & 7] = fmaxf(mxv[e & 7], __uint_as_float(s[e]));
      } else {
#pragma unroll
        for (int e = 0; e < 64; e += 2)
          mxv[(e >> 1) & 7] = fmax3(mxv[(e >> 1) & 7], __uint_as_float(s[e]), __uint_as_float(s[e + 1]));
      }
      const float mx = fmaxf(fmaxf(fmaxf(mxv[0], mxv[1]), fmaxf(mxv[2], mxv[3])),
                             fmaxf(fmaxf(mxv[4], mxv[5]), fmaxf(mxv[6], mxv[7])));
      // Exact running max (of this half): the largest term so far gets
      // p = 1, which bf16 holds exactly.  (A stale max, as lazy rescaling
      // keeps, would round that dominant term by up to 2^-9, and the error
      // would reach D = rowsum(dO * O) of the backward unscaled.)  A half
      // whose columns are all masked so far keeps m = -inf and p = 0.
      const float m_new = fmaxf(m_used, mx * scale_log2);
      const bool grow = m_new > m_used;
      const float alpha = grow ? ex2(m_used - m_new) : 1.f;
      m_used = m_new;
      const float m_sub = m_used == -INFINITY ? 0.f : m_used;
      // x = s scale - m and the row sum in packed fp32 pairs
      const uint64_t sc2 = f2_pack(scale_log2, scale_log2), nm2 = f2_pack(-m_sub, -m_sub);
      uint64_t rs2[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) rs2[u] = f2_pack(0.f, 0.f);
      // two copies of the loop, so that unmasked tiles (all but one) carry no
      // per-column compare
      auto exp_tile = [&](auto masked) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t pk[8];
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            const int i = c * 16 + e;
            const float2 x = f2_unpack(f2_fma(f2_pack(__uint_as_float(s[i]), __uint_as_float(s[i + 1])), sc2, nm2));
            float p0 = ex2(x.x), p1 = ex2(x.y);
            if constexpr (decltype(masked)::value) {
              p0 = (c0 + i < lim) ? p0 : 0.f;
              p1 = (c0 + i + 1 < lim) ? p1 : 0.f;
            }
            rs2[(i >> 1) & 3] = f2_add(rs2[(i >> 1) & 3], f2_pack(p0, p1));
            pk[e >> 1] = pack_bf16x2(p0, p1);
          }
          // P of columns 16 c .. 16 c + 15 of this half lands on columns
          // 8 c .. 8 c + 7, whose scores were read above
          tmem_st8(tS + c * 8, pk);
        }
      };
      if (msk) exp_tile(std::true_type{});
      else exp_tile(std::false_type{});
      const float2 ra = f2_unpack(f2_add(rs2[0], rs2[1])), rb = f2_unpack(f2_add(rs2[2], rs2[3]));
      const float rs = (ra.x + ra.y) + (rb.x + rb.y);
      lsum = lsum * alpha + rs;
      // O_h holds P_h V_h of the earlier tiles; bring it to the new max once
      // P(j - 1) V(j - 1) has finished.
      if (j > 0 && __any_sync(0xffffffffu, grow)) {
        if (!mbar_wait_w(&bars->pvdone[(j - 1) & 1], ((j - 1) >> 1) & 1, status, 9)) { ok = false; break; }
        tc_fence_after();
        const uint64_t a2 = f2_pack(alpha, alpha);
#pragma unroll
        for (int c = 0; c < HD / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + c * 32, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; e += 2) {   // packed pairs: half the multiplies
            const float2 y = f2_unpack(f2_mul(f2_pack(__uint_as_float(o[e]), __uint_as_float(o[e + 1])), a2));
            o[e] = __float_as_uint(y.x);
            o[e + 1] = __float_as_uint(y.y);
          }
          tmem_st32(tO + c * 32, o);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars->pfull[b][h]);
    }
    // ---- merge the two halves; warpgroup h writes output columns
    // HD/2 h .. HD/2 h + HD/2 - 1
    float2* mg = reinterpret_cast<float2*>(smem + Lay::merge);
    mg[h * BM + r] = make_float2(m_used, lsum);
    const bool chain = !(first && last);             // a ring step that merges
    const int64_t row_off = (int64_t)bh * S + qrow;
    const float lse2_a = (chain && !first && qrow < S) ? lse2_acc[row_off] : -INFINITY;
    named_bar(1, 2 * kHalf);                         // both halves have read lse2_acc
    const float2 o_ml = mg[(h ^ 1) * BM + r];
    if (ok && mbar_wait_w(&bars->pvdone[(n_kv - 1) & 1], ((n_kv - 1) >> 1) & 1, status, 10)) {
      tc_fence_after();
      const float m0 = h ? o_ml.x : m_used, l0 = h ? o_ml.y : lsum;
      const float m1 = h ? m_used : o_ml.x, l1 = h ? lsum : o_ml.y;
      const float m = fmaxf(m0, m1);                 // finite: column 0 is never masked
      const float a0 = ex2(m0 - m), a1 = ex2(m1 - m);
      const float l = l0 * a0 + l1 * a1;
      const float inv = 1.f / l;
      float w0 = a0 * inv, w1 = a1 * inv;
      // ring step: weights of the accumulated and of this block's output
      float lse2_out = m + __log2f(l), fa = 0.f;
      if (chain) {
        const float b = lse2_out;
        const float mx = fmaxf(lse2_a, b);
        const float wa = first ? 0.f : ex2(lse2_a - mx), wb = ex2(b - mx);
        const float z = wa + wb;
        lse2_out = mx + __log2f(z);
        fa = wa / z;
        w0 *= wb / z;
        w1 *= wb / z;
      }
      const uint32_t tO0 = tmem + lane_addr + 256, tO1 = tO0 + HD;
#pragma unroll
      for (int cc = 0; cc < HD / 64; ++cc) {
        const int c = h * (HD / 64) + cc;            // 32-column chunk of the output
        uint32_t o0[32], o1[32];
        tmem_ld32(tO0 + c * 32, o0);
        tmem_ld32(tO1 + c * 32, o1);
        tmem_ld_wait();
        if (qrow < S) {
          const int64_t base = ((int64_t)bh * S + qrow) * (HD / 8) + c * 4;
          float4* acc = chain ? reinterpret_cast<float4*>(o_acc) + row_off * (HD / 4) + c * 8
                              : nullptr;
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            float xv[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
              xv[e] = __uint_as_float(o0[v * 8 + e]) * w0 + __uint_as_float(o1[v * 8 + e]) * w1;
            if (chain && !first) {
              const float4 a = acc[2 * v], b = acc[2 * v + 1];
              xv[0] += fa * a.x; xv[1] += fa * a.y; xv[2] += fa * a.z; xv[3] += fa * a.w;
              xv[4] += fa * b.x; xv[5] += fa * b.y; xv[6] += fa * b.z; xv[7] += fa * b.w;
            }
            if (!last) {                             // keep the merged fp32 output
              acc[2 * v] = make_float4(xv[0], xv[1], xv[2], xv[3]);
              acc[2 * v + 1] = make_float4(xv[4], xv[5], xv[6], xv[7]);
              continue;
            }
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
      if (h == 0 && qrow < S) {
        if (last) lse[row_off] = lse2_out * 0.69314718055994531f;
        else lse2_acc[row_off] = lse2_out;
      }
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

// cuTensorMapEncodeTiled from the driver, looked up once.
PFN_cuTensorMapEncodeTiled_v12000 lh_tensormap_encoder() { return get_encode(); }

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
                               lh_bf16* og_lo, float* lse, int* status, cudaStream_t st,
                               int full, int first, int last, float* o_acc, float* lse2_acc) {
  CUtensorMap tq, tk, tv;
  if (!lh_make_tmap_3d(&tq, qg, BH, S, d, BM) || !lh_make_tmap_3d(&tk, kg, BH, S, d, BN) ||
      !lh_make_tmap_3d(&tv, vg, BH, S, d, BN))
    return cudaErrorInvalidValue;
  const int n_qt = (int)((S + BM - 1) / BM);
  const dim3 grid((unsigned)(n_qt * BH));
  const float scale_log2 = scale * 1.4426950408889634f;
  if (d == 128) {
    cudaFuncSetAttribute(k_attn_fwd<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    k_attn_fwd<128><<<grid, kThreads, kSmemBytes, st>>>(tq, tk, tv, (uint4*)og, (uint4*)og_lo, lse,
                                                         (int)S, BH, scale_log2, status, full,
                                                         first, last, o_acc, lse2_acc);
  } else if (d == 64) {
    cudaFuncSetAttribute(k_attn_fwd<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    k_attn_fwd<64><<<grid, kThreads, kSmemBytes, st>>>(tq, tk, tv, (uint4*)og, (uint4*)og_lo, lse,
                                                        (int)S, BH, scale_log2, status, full,
                                                        first, last, o_acc, lse2_acc);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}
