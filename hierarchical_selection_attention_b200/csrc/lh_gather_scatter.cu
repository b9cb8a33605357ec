// Data movement around the attention of Lighthouse Attention ("Long Context
// Pre-Training with Lighthouse Attention", Sec. 3.5 gather, Sec. 3.6
// scatter-back) and the adjoints of both (Sec. 3.2: gradients flow through
// the scatter, the attention and the gather).
//
// All kernels are HBM-bound.  One thread moves one 16-byte vector (8 bf16
// features) of one row; consecutive threads take consecutive vectors of a
// row, so warp accesses are whole 256-byte (d = 128) or 128-byte (d = 64)
// rows, and index loads are shared by the d/8 threads of a row.  Sums run in
// fp32 in a fixed order (ascending level, ascending token) and are rounded
// once to bf16, so every output is deterministic.
#include "lh_common.cuh"

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ void acc8(float* a, const uint4& u, float s = 1.f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = unpack_bf16x2(w[e]);
    a[2 * e] = fmaf(f.x, s, a[2 * e]);
    a[2 * e + 1] = fmaf(f.y, s, a[2 * e + 1]);
  }
}

__device__ __forceinline__ uint4 pack8(const float* a) {
  uint4 u;
  u.x = pack_bf16x2(a[0], a[1]);
  u.y = pack_bf16x2(a[2], a[3]);
  u.z = pack_bf16x2(a[4], a[5]);
  u.w = pack_bf16x2(a[6], a[7]);
  return u;
}

// Vector index of row (b, i, h) of level l in the pyramid: level 0 is the
// input tensor, level l >= 1 lives in the pooled buffer.
__device__ __forceinline__ const uint4* level_row(const LhDims& D, const uint4* x0,
                                                  const uint4* xl, int l, int b, int64_t i,
                                                  int h, int V) {
  if (l == 0) return x0 + (((int64_t)b * D.N + i) * D.H + h) * V;
  return xl + (((int64_t)D.B * D.pool_row[l] + (int64_t)b * D.lvl_size[l] + i) * D.H + h) * V;
}

// (iii) gather: thread = (b, h, slot m, vector cv).  I is the index type:
// 32-bit whenever the item count fits, which keeps the div/mod cheap.
template <typename I>
__global__ void __launch_bounds__(kThreads) k_gather(LhDims D, const uint4* __restrict__ q,
                                                     const uint4* __restrict__ k,
                                                     const uint4* __restrict__ v,
                                                     const uint4* __restrict__ q_lv,
                                                     const uint4* __restrict__ k_lv,
                                                     const uint4* __restrict__ v_lv,
                                                     const int32_t* __restrict__ sel_idx,
                                                     uint4* __restrict__ qg, uint4* __restrict__ kg,
                                                     uint4* __restrict__ vg) {
  const int V = D.d >> 3;
  const I item = (I)blockIdx.x * blockDim.x + threadIdx.x;
  const I total = (I)D.B * D.H * D.S * V;
  if (item >= total) return;
  const int cv = (int)(item & (V - 1));
  const I row = item / V;  // (bh, m)
  const I bh = row / (I)D.S;
  const int b = (int)(bh / D.H), h = (int)(bh % D.H);
  const int64_t f = __ldg(sel_idx + row);
  if (f < 0 || f >= D.P) {
    lh_report(D.status, LH_ERR_DEVICE_BOUNDS, 200);
    return;
  }
  const int l = lh_level_of(D, f);
  const int64_t i = f - D.lvl_off[l];
  const int64_t o = (int64_t)row * V + cv;
  qg[o] = __ldg(level_row(D, q, q_lv, l, b, i, h, V) + cv);
  kg[o] = __ldg(level_row(D, k, k_lv, l, b, i, h, V) + cv);
  vg[o] = __ldg(level_row(D, v, v_lv, l, b, i, h, V) + cv);
}

// Tokens a thread of k_scatter / k_gather_bwd takes: G divides p (and N), so
// the G tokens of an aligned group share their entry at every level l >= 1,
// and each thread turns two memory round trips (slot lookups, then rows) into
// G output rows instead of one.
constexpr int kMaxG = 4;

// (iv) scatter-back, gather side: thread = (b, group g, h, vector cv), where
// group g holds the tokens t with t + 1 in [gG, gG + G).  The entry of level l
// that reaches t is i = floor((t+1)/p^l) - 1, the same for the whole group at
// every l >= 1; level 0 contributes entry t itself.  All slot lookups are
// issued before any row load, and all row loads before the sums; each row is
// summed in ascending level order.
template <int L, typename I>
__global__ void __launch_bounds__(kThreads, 6) k_scatter(LhDims D, int G, I NG,
                                                      const uint4* __restrict__ og,
                                                      const int32_t* __restrict__ slot_map,
                                                      uint4* __restrict__ o) {
  constexpr int LC = L > 1 ? L - 1 : 1;
  const int V = D.d >> 3;
  const I item = (I)blockIdx.x * blockDim.x + threadIdx.x;
  const I total = (I)D.B * NG * D.H * V;
  if (item >= total) return;
  const int cv = (int)(item & (V - 1));
  const I r = item / V;  // (b, g, h)
  const int h = (int)(r % (I)D.H);
  const I bg = r / (I)D.H;
  const int64_t j0 = (int64_t)(bg % NG) * G;  // t + 1 of the group's first token
  const int b = (int)(bg / NG);
  const int64_t bh = (int64_t)b * D.H + h;
  const int32_t* sm = slot_map + bh * D.P;
  const uint4* src = og + bh * D.S * V + cv;
  int cslot[LC], fslot[kMaxG];
#pragma unroll
  for (int l = 1; l < L; ++l) {
    const int64_t j = j0 / D.lvl_span[l];
    cslot[l - 1] = j ? __ldg(sm + D.lvl_off[l] + j - 1) : -1;
  }
#pragma unroll
  for (int u = 0; u < kMaxG; ++u) {
    const int64_t t = j0 - 1 + u;
    fslot[u] = (u < G && t >= 0 && t < D.N) ? __ldg(sm + D.lvl_off[0] + t) : -1;
  }
  uint4 crow[LC], frow[kMaxG];
#pragma unroll
  for (int l = 1; l < L; ++l)
    if (cslot[l - 1] >= 0) crow[l - 1] = __ldg(src + (int64_t)cslot[l - 1] * V);
#pragma unroll
  for (int u = 0; u < kMaxG; ++u)
    if (fslot[u] >= 0) frow[u] = __ldg(src + (int64_t)fslot[u] * V);
#pragma unroll
  for (int u = 0; u < kMaxG; ++u) {
    const int64_t t = j0 - 1 + u;
    if (u >= G || t < 0 || t >= D.N) continue;
    float a[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (fslot[u] >= 0) acc8(a, frow[u]);
#pragma unroll
    for (int l = 1; l < L; ++l)
      if (cslot[l - 1] >= 0) acc8(a, crow[l - 1]);
    o[(((int64_t)b * D.N + t) * D.H + h) * V + cv] = pack8(a);
  }
}

// (iv) in fixed-point integer atomics: every selected entry adds its output,
// scaled by 2^32 and rounded to an integer, into the 64-bit accumulators of
// its shifted range; integer addition is associative, so the sums do not
// depend on the order the atomics land in.  Thread = (b, h, entry f, pair of
// features); unselected entries leave at once.
__global__ void __launch_bounds__(kThreads) k_scatter_push(LhDims D, const uint32_t* __restrict__ og,
                                                           const int32_t* __restrict__ slot_map,
                                                           unsigned long long* __restrict__ acc) {
  const int Vp = D.d >> 1;  // bf16 pairs per row
  const int64_t item = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t total = (int64_t)D.B * D.H * D.P * Vp;
  if (item >= total) return;
  const int c2 = (int)(item % Vp);
  const int64_t ent = item / Vp;        // (bh, f)
  const int64_t bh = ent / D.P;
  const int64_t f = ent % D.P;
  const int slot = __ldg(slot_map + ent);
  if (slot < 0) return;
  const int b = (int)(bh / D.H), h = (int)(bh % D.H);
  const int l = lh_level_of(D, f);
  const int64_t i = f - D.lvl_off[l];
  const int64_t span = D.lvl_span[l];
  const int64_t start = (i + 1) * span - 1;
  const int64_t stop = min(start + span, D.N);
  const float2 x = unpack_bf16x2(__ldg(og + (bh * D.S + slot) * Vp + c2));
  const long long ix = __double2ll_rn((double)x.x * 4294967296.0);
  const long long iy = __double2ll_rn((double)x.y * 4294967296.0);
  for (int64_t t = start; t < stop; ++t) {
    unsigned long long* dst = acc + (((int64_t)b * D.N + t) * D.H + h) * D.d + 2 * c2;
    atomicAdd(dst, (unsigned long long)ix);
    atomicAdd(dst + 1, (unsigned long long)iy);
  }
}

__global__ void __launch_bounds__(kThreads) k_scatter_fix2bf16(int64_t n,
                                                               const long long* __restrict__ acc,
                                                               uint32_t* __restrict__ o) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float a = (float)((double)acc[2 * i] * (1.0 / 4294967296.0));
  const float b = (float)((double)acc[2 * i + 1] * (1.0 / 4294967296.0));
  o[i] = pack_bf16x2(a, b);
}

// Adjoint of the scatter, fused with D = rowsum(dog * og): thread = (b, h,
// slot m, vector cv); it sums dO over the shifted range of the slot's entry.
template <typename I>
__global__ void __launch_bounds__(kThreads) k_scatter_bwd(LhDims D, const uint4* __restrict__ dout,
                                                          const uint4* __restrict__ og,
                                                          const uint4* __restrict__ og_lo,
                                                          const int32_t* __restrict__ sel_idx,
                                                          uint4* __restrict__ dog,
                                                          float* __restrict__ delta) {
  const int V = D.d >> 3;
  const I item = (I)blockIdx.x * blockDim.x + threadIdx.x;
  const I total = (I)D.B * D.H * D.S * V;
  const unsigned live = __ballot_sync(0xffffffffu, item < total);
  if (item >= total) return;
  const int cv = (int)(item & (V - 1));
  const I row = item / V;
  const I bh = row / (I)D.S;
  const int b = (int)(bh / D.H), h = (int)(bh % D.H);
  const int64_t f = __ldg(sel_idx + row);
  const int l = lh_level_of(D, f);
  const int64_t i = f - D.lvl_off[l];
  const int64_t span = D.lvl_span[l];
  const int64_t start = (i + 1) * span - 1;
  const int64_t stop = min(start + span, D.N);
  const int64_t HV = (int64_t)D.H * V;
  const uint4* src = dout + ((int64_t)b * D.N * D.H + h) * V + cv;
  float a[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  int64_t t = start;
  for (; t + 4 <= stop; t += 4) {
    const uint4 u0 = __ldg(src + t * HV), u1 = __ldg(src + (t + 1) * HV);
    const uint4 u2 = __ldg(src + (t + 2) * HV), u3 = __ldg(src + (t + 3) * HV);
    acc8(a, u0); acc8(a, u1); acc8(a, u2); acc8(a, u3);
  }
  for (; t < stop; ++t) acc8(a, __ldg(src + t * HV));
  const uint4 packed = pack8(a);
  dog[item] = packed;
  // D with dO~ as the attention backward sees it (rounded) and the output
  // to ~16 bits (og + og_lo): D feeds dS = P (dP - D) unscaled, so an error
  // of one bf16 rounding in O would pass straight into the gradients.
  float rd[8] = {0, 0, 0, 0, 0, 0, 0, 0}, ro[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  acc8(rd, packed);
  acc8(ro, __ldg(og + item));
  if (og_lo) acc8(ro, __ldg(og_lo + item));
  float s = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) s = fmaf(rd[e], ro[e], s);
  for (int o = V >> 1; o > 0; o >>= 1) s += __shfl_xor_sync(live, s, o);
  if (cv == 0) delta[row] = s;
}

// D = rowsum(dog * (og + og_lo)) for the standalone attention backward.
__global__ void __launch_bounds__(kThreads) k_attn_delta(int64_t rows, int V,
                                                         const uint4* __restrict__ og,
                                                         const uint4* __restrict__ og_lo,
                                                         const uint4* __restrict__ dog,
                                                         float* __restrict__ delta) {
  const int64_t item = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const unsigned live = __ballot_sync(0xffffffffu, item < rows * V);
  if (item >= rows * V) return;
  float rd[8] = {0, 0, 0, 0, 0, 0, 0, 0}, ro[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  acc8(rd, __ldg(dog + item));
  acc8(ro, __ldg(og + item));
  if (og_lo) acc8(ro, __ldg(og_lo + item));
  float s = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) s = fmaf(rd[e], ro[e], s);
  for (int o = V >> 1; o > 0; o >>= 1) s += __shfl_xor_sync(live, s, o);
  if (item % V == 0) delta[item / V] = s;
}

// Adjoint of gather + mean pooling: thread = (b, group g, h, vector cv),
// group g holding the tokens t in [gG, gG + G).  The level-l entry whose
// (unshifted) window holds t is i = floor(t / p^l), the same for the whole
// group at every l >= 1.  Slot lookups first, then every row load, then the
// sums, each in ascending level order (two memory round trips per G rows).
// The level-0 rows of the selected tokens (few: most tokens are reached only
// through coarser entries) are copied into the thread's own shared-memory
// slots with cp.async instead of being held in registers, which leaves room
// for three blocks per SM.
constexpr size_t kGatherBwdSmem = (size_t)kMaxG * 3 * kThreads * sizeof(uint4);   // 48 KB

template <int L, typename I>
__global__ void __launch_bounds__(kThreads, L <= 4 ? 3 : 1)
    k_gather_bwd(LhDims D, int G, I NG, const uint4* __restrict__ dqg,
                 const uint4* __restrict__ dkg, const uint4* __restrict__ dvg,
                 const int32_t* __restrict__ slot_map, uint4* __restrict__ dq,
                 uint4* __restrict__ dk, uint4* __restrict__ dv) {
  extern __shared__ uint4 fine[];   // [kMaxG][3][blockDim.x]
  constexpr int LC = L > 1 ? L - 1 : 1;
  const int V = D.d >> 3;
  const I item = (I)blockIdx.x * blockDim.x + threadIdx.x;
  const I total = (I)D.B * NG * D.H * V;
  if (item >= total) return;
  const int cv = (int)(item & (V - 1));
  const I r = item / V;
  const int h = (int)(r % (I)D.H);
  const I bg = r / (I)D.H;
  const int64_t t0 = (int64_t)(bg % NG) * G;
  const int b = (int)(bg / NG);
  const int64_t bh = (int64_t)b * D.H + h;
  const int32_t* sm = slot_map + bh * D.P;
  const int64_t base = bh * D.S * V + cv;
  const unsigned nt = blockDim.x;
  uint4* mine = fine + threadIdx.x;
  int cslot[LC], fslot[kMaxG];
#pragma unroll
  for (int l = 1; l < L; ++l) cslot[l - 1] = __ldg(sm + D.lvl_off[l] + t0 / D.lvl_span[l]);
#pragma unroll
  for (int u = 0; u < kMaxG; ++u) fslot[u] = u < G ? __ldg(sm + D.lvl_off[0] + t0 + u) : -1;
#pragma unroll
  for (int u = 0; u < kMaxG; ++u) {
    if (fslot[u] >= 0) {
      const int64_t s = base + (int64_t)fslot[u] * V;
      lh_cp_async16(mine + (u * 3 + 0) * nt, dqg + s);
      lh_cp_async16(mine + (u * 3 + 1) * nt, dkg + s);
      lh_cp_async16(mine + (u * 3 + 2) * nt, dvg + s);
    }
  }
  lh_cp_async_commit();
  uint4 cq[LC], ck[LC], cvv[LC];
#pragma unroll
  for (int l = 1; l < L; ++l) {
    if (cslot[l - 1] >= 0) {
      const int64_t s = base + (int64_t)cslot[l - 1] * V;
      cq[l - 1] = __ldg(dqg + s);
      ck[l - 1] = __ldg(dkg + s);
      cvv[l - 1] = __ldg(dvg + s);
    }
  }
  lh_cp_async_wait<0>();
#pragma unroll
  for (int u = 0; u < kMaxG; ++u) {
    if (u >= G) continue;
    float aq[8] = {0, 0, 0, 0, 0, 0, 0, 0}, ak[8] = {0, 0, 0, 0, 0, 0, 0, 0},
          av[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (fslot[u] >= 0) {
      acc8(aq, mine[(u * 3 + 0) * nt]);
      acc8(ak, mine[(u * 3 + 1) * nt]);
      acc8(av, mine[(u * 3 + 2) * nt]);
    }
#pragma unroll
    for (int l = 1; l < L; ++l) {
      if (cslot[l - 1] < 0) continue;
      const float w = 1.f / (float)D.lvl_span[l];
      acc8(aq, cq[l - 1], w);
      acc8(ak, ck[l - 1], w);
      acc8(av, cvv[l - 1], w);
    }
    const int64_t o = (((int64_t)b * D.N + t0 + u) * D.H + h) * V + cv;
    dq[o] = pack8(aq);
    dk[o] = pack8(ak);
    dv[o] = pack8(av);
  }
}

inline unsigned nblocks(int64_t n) { return (unsigned)((n + kThreads - 1) / kThreads); }

constexpr int64_t kIdx32 = (int64_t)1 << 31;  // item counts below this use 32-bit indices

template <typename I>
cudaError_t scatter_L(const LhDims& D, unsigned g, int G, I NG, const uint4* x, const int32_t* sm,
                      uint4* o, cudaStream_t st) {
  switch (D.L) {
    case 1: k_scatter<1, I><<<g, kThreads, 0, st>>>(D, G, NG, x, sm, o); break;
    case 2: k_scatter<2, I><<<g, kThreads, 0, st>>>(D, G, NG, x, sm, o); break;
    case 3: k_scatter<3, I><<<g, kThreads, 0, st>>>(D, G, NG, x, sm, o); break;
    case 4: k_scatter<4, I><<<g, kThreads, 0, st>>>(D, G, NG, x, sm, o); break;
    case 5: k_scatter<5, I><<<g, kThreads, 0, st>>>(D, G, NG, x, sm, o); break;
    case 6: k_scatter<6, I><<<g, kThreads, 0, st>>>(D, G, NG, x, sm, o); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

template <typename I>
cudaError_t gather_bwd_L(const LhDims& D, unsigned g, int G, I NG, const uint4* a, const uint4* b,
                         const uint4* c, const int32_t* sm, uint4* x, uint4* y, uint4* z,
                         cudaStream_t st) {
  switch (D.L) {
    case 1: k_gather_bwd<1, I><<<g, kThreads, kGatherBwdSmem, st>>>(D, G, NG, a, b, c, sm, x, y, z); break;
    case 2: k_gather_bwd<2, I><<<g, kThreads, kGatherBwdSmem, st>>>(D, G, NG, a, b, c, sm, x, y, z); break;
    case 3: k_gather_bwd<3, I><<<g, kThreads, kGatherBwdSmem, st>>>(D, G, NG, a, b, c, sm, x, y, z); break;
    case 4: k_gather_bwd<4, I><<<g, kThreads, kGatherBwdSmem, st>>>(D, G, NG, a, b, c, sm, x, y, z); break;
    case 5: k_gather_bwd<5, I><<<g, kThreads, kGatherBwdSmem, st>>>(D, G, NG, a, b, c, sm, x, y, z); break;
    case 6: k_gather_bwd<6, I><<<g, kThreads, kGatherBwdSmem, st>>>(D, G, NG, a, b, c, sm, x, y, z); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

// G of k_scatter / k_gather_bwd: the largest of 4, 2, 1 that divides p (for
// L > 1, p^(L-1) divides N, so G divides N too) or, for L = 1, N.
inline int token_group(const LhDims& D) {
  const int64_t m = D.L > 1 ? D.p : D.N;
  return m % 4 == 0 ? 4 : (m % 2 == 0 ? 2 : 1);
}

}  // namespace

cudaError_t lh_launch_gather(const LhDims& D, const lh_bf16* q, const lh_bf16* k,
                             const lh_bf16* v, const lh_bf16* q_lv, const lh_bf16* k_lv,
                             const lh_bf16* v_lv, const int32_t* sel_idx, lh_bf16* qg,
                             lh_bf16* kg, lh_bf16* vg, cudaStream_t st) {
  const int64_t n = (int64_t)D.B * D.H * D.S * (D.d >> 3);
  if (n < kIdx32)
    k_gather<uint32_t><<<nblocks(n), kThreads, 0, st>>>(
        D, (const uint4*)q, (const uint4*)k, (const uint4*)v, (const uint4*)q_lv,
        (const uint4*)k_lv, (const uint4*)v_lv, sel_idx, (uint4*)qg, (uint4*)kg, (uint4*)vg);
  else
    k_gather<uint64_t><<<nblocks(n), kThreads, 0, st>>>(
        D, (const uint4*)q, (const uint4*)k, (const uint4*)v, (const uint4*)q_lv,
        (const uint4*)k_lv, (const uint4*)v_lv, sel_idx, (uint4*)qg, (uint4*)kg, (uint4*)vg);
  return cudaGetLastError();
}

cudaError_t lh_launch_scatter(const LhDims& D, const lh_bf16* og, const int32_t* slot_map,
                              lh_bf16* o, cudaStream_t st) {
  const int G = token_group(D);
  const int64_t NG = D.N / G + 1;  // shifted groups: t + 1 runs over 1..N
  const int64_t n = (int64_t)D.B * NG * D.H * (D.d >> 3);
  const unsigned g = nblocks(n);
  const uint4* x = (const uint4*)og;
  if (n < kIdx32) return scatter_L<uint32_t>(D, g, G, (uint32_t)NG, x, slot_map, (uint4*)o, st);
  return scatter_L<uint64_t>(D, g, G, (uint64_t)NG, x, slot_map, (uint4*)o, st);
}

size_t lh_scatter_atomic_ws_bytes(const LhDims& D) {
  return (size_t)D.B * D.N * D.H * D.d * sizeof(long long);
}

cudaError_t lh_launch_scatter_atomic(const LhDims& D, const lh_bf16* og,
                                     const int32_t* slot_map, lh_bf16* o, void* ws,
                                     cudaStream_t st, int* launches) {
  const int64_t elems = (int64_t)D.B * D.N * D.H * D.d;
  cudaError_t e = cudaMemsetAsync(ws, 0, (size_t)elems * sizeof(long long), st);
  if (e != cudaSuccess) return e;
  const int64_t n = (int64_t)D.B * D.H * D.P * (D.d >> 1);
  k_scatter_push<<<nblocks(n), kThreads, 0, st>>>(D, (const uint32_t*)og, slot_map,
                                                  (unsigned long long*)ws);
  k_scatter_fix2bf16<<<nblocks(elems / 2), kThreads, 0, st>>>(elems / 2, (const long long*)ws,
                                                             (uint32_t*)o);
  if (launches) *launches = 2;
  return cudaGetLastError();
}

cudaError_t lh_launch_scatter_bwd(const LhDims& D, const lh_bf16* dout, const lh_bf16* og,
                                  const lh_bf16* og_lo, const int32_t* sel_idx, lh_bf16* dog,
                                  float* delta, cudaStream_t st) {
  const int64_t n = (int64_t)D.B * D.H * D.S * (D.d >> 3);
  if (n < kIdx32)
    k_scatter_bwd<uint32_t><<<nblocks(n), kThreads, 0, st>>>(
        D, (const uint4*)dout, (const uint4*)og, (const uint4*)og_lo, sel_idx, (uint4*)dog, delta);
  else
    k_scatter_bwd<uint64_t><<<nblocks(n), kThreads, 0, st>>>(
        D, (const uint4*)dout, (const uint4*)og, (const uint4*)og_lo, sel_idx, (uint4*)dog, delta);
  return cudaGetLastError();
}

cudaError_t lh_launch_attn_delta(int BH, int64_t S, int d, const lh_bf16* og,
                                 const lh_bf16* og_lo, const lh_bf16* dog, float* delta,
                                 cudaStream_t st) {
  const int64_t rows = (int64_t)BH * S;
  k_attn_delta<<<nblocks(rows * (d >> 3)), kThreads, 0, st>>>(rows, d >> 3, (const uint4*)og,
                                                             (const uint4*)og_lo,
                                                             (const uint4*)dog, delta);
  return cudaGetLastError();
}

cudaError_t lh_launch_gather_bwd(const LhDims& D, const lh_bf16* dqg, const lh_bf16* dkg,
                                 const lh_bf16* dvg, const int32_t* slot_map, lh_bf16* dq,
                                 lh_bf16* dk, lh_bf16* dv, cudaStream_t st) {
  const int G = token_group(D);
  const int64_t NG = D.N / G;
  const int64_t n = (int64_t)D.B * NG * D.H * (D.d >> 3);
  const unsigned g = nblocks(n);
  const uint4 *a = (const uint4*)dqg, *b = (const uint4*)dkg, *c = (const uint4*)dvg;
  uint4 *x = (uint4*)dq, *y = (uint4*)dk, *z = (uint4*)dv;
  if (n < kIdx32)
    return gather_bwd_L<uint32_t>(D, g, G, (uint32_t)NG, a, b, c, slot_map, x, y, z, st);
  return gather_bwd_L<uint64_t>(D, g, G, (uint64_t)NG, a, b, c, slot_map, x, y, z, st);
}
