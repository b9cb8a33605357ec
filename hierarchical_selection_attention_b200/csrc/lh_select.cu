// Stage (ii) selection and the topological order of stage (iii)
// ("Long Context Pre-Training with Lighthouse Attention", Sec. 3.4 and 3.5).
//
// Joint top-k.  Every finer-level entry f (levels 0..L-2) gets the unique
// 64-bit key
//      key(f) = bits(max(QK_f, KQ_f)) << 32  |  (2^32 - 1 - f)
// (scores are >= 0, so their fp32 bit patterns order like the values, and the
// low word makes the lower flat index win a tie).  Taking distinct entries
// from the QK and KQ streams merged by score is the same as taking the n_sel
// largest keys, because an entry first shows up at the larger of its two
// scores.  The n_sel-th largest key is found by radix selection, 11 bits per
// pass from the top: a histogram pass counts the digits of the keys that
// still match the prefix found so far, and a one-block pass picks the digit
// that holds the n_sel-th key.  Once every key left in that digit is needed,
// the threshold is final and later passes return at once.  Then
// selected(f) <=> key(f) >= threshold: integer work only, so the selected
// set is bit-exact and the same on every run.
//
// Selection modes.  Mode 0 runs that selection once over all finer entries
// (n_sel to take); mode 1, the per-level quota, runs it once per finer level
// (p k to take from each, Eq. 8 read as an exact per-level count).  Each run
// is a "segment" with its own histograms, state and threshold.  Mode 2, the
// stratified selection, cuts the candidates into n_sel / m contiguous chunks
// and keeps the top m of each; a chunk is small (about m C / n_sel keys), so
// one block runs all of its radix passes with the histogram in shared memory
// and keeps only the final threshold.
//
// Order.  Entries are sorted by the last base token they summarise,
// e = (i+1) p^l - 1, and by level.  Walking the base tokens t in order and,
// for each, the levels whose entries end at t ((t+1) mod p^l == 0) in
// ascending order lists the selected entries in exactly that order, so slots
// come from a prefix sum over t of the number of selected entries ending at
// t: a counting pass per block of tokens, a scan over blocks, and an emit
// pass that writes sel_idx (slot -> entry) and slot_map (entry -> slot or -1).
#include <cub/block/block_reduce.cuh>
#include <cub/block/block_scan.cuh>

#include "lh_common.cuh"

namespace {

constexpr int kPasses = 6;
constexpr int kBins = 2048;
__constant__ int c_shift[kPasses] = {53, 42, 31, 20, 9, 0};
__constant__ int c_width[kPasses] = {11, 11, 11, 11, 11, 9};

struct SelState {
  unsigned long long prefix;  // digits fixed so far (lower bits zero)
  long long need;             // keys still to take among those matching prefix
  int done;                   // threshold final
  int pad;
};

constexpr int kOrderThreads = 256;
constexpr int kOrderItems = 4;                        // tokens per thread
constexpr int kOrderTile = kOrderThreads * kOrderItems;

__device__ __forceinline__ unsigned long long entry_key(const float* qk, const float* kq,
                                                        int64_t f) {
  const float r = fmaxf(__ldg(qk + f), __ldg(kq + f));
  return ((unsigned long long)__float_as_uint(r) << 32) |
         (unsigned long long)(0xffffffffu - (uint32_t)f);
}

__global__ void __launch_bounds__(256) k_sel_hist(LhDims D, const float* __restrict__ qk,
                                                  const float* __restrict__ kq,
                                                  unsigned* __restrict__ hist,
                                                  const SelState* __restrict__ state, int pass) {
  const int64_t bs = blockIdx.y;                // (b, h) x segment
  const int64_t bh = bs / D.nseg;
  const int seg = (int)(bs - bh * D.nseg);
  unsigned long long prefix = 0;
  if (pass > 0) {
    const SelState s = state[bs];
    if (s.done) return;
    prefix = s.prefix;
  }
  __shared__ unsigned h[kBins];
  for (int i = threadIdx.x; i < kBins; i += blockDim.x) h[i] = 0;
  __syncthreads();
  const int shift = c_shift[pass];
  const int hi = shift + c_width[pass];
  const unsigned mask = (1u << c_width[pass]) - 1u;
  const float* q = qk + bh * D.P;
  const float* k = kq + bh * D.P;
  const int64_t seg_end = D.seg_lo[seg] + D.seg_len[seg];
  const int64_t per_block = (D.seg_len[seg] + gridDim.x - 1) / gridDim.x;
  const int64_t lo = D.seg_lo[seg] + (int64_t)blockIdx.x * per_block;
  const int64_t end = min(lo + per_block, seg_end);
  const int64_t span = end > lo ? end - lo : 0;
  const int64_t rounds = (span + blockDim.x - 1) / blockDim.x;
  for (int64_t r = 0; r < rounds; ++r) {
    const int64_t f = lo + r * blockDim.x + threadIdx.x;
    bool in = f < end;
    unsigned digit = 0;
    if (in) {
      const unsigned long long key = entry_key(q, k, f);
      in = (hi >= 64) || ((key >> hi) == (prefix >> hi));
      digit = (unsigned)(key >> shift) & mask;
    }
    // warp-aggregated increment: one shared atomic per distinct digit
    const unsigned act = __ballot_sync(0xffffffffu, in);
    if (in) {
      const unsigned peers = __match_any_sync(act, digit);
      if ((threadIdx.x & 31) == (unsigned)(__ffs(peers) - 1)) atomicAdd(&h[digit], __popc(peers));
    }
  }
  __syncthreads();
  unsigned* g = hist + (bs * kPasses + pass) * kBins;
  for (int i = threadIdx.x; i < kBins; i += blockDim.x)
    if (h[i]) atomicAdd(&g[i], h[i]);
}

// One block of 256 threads per (b, h) and segment; thread t owns digits
// 2047-8t .. 2040-8t.
__global__ void __launch_bounds__(256) k_sel_find(LhDims D, const unsigned* __restrict__ hist,
                                                  SelState* __restrict__ state, int pass) {
  const int64_t bh = blockIdx.x;                 // (b, h) x segment
  SelState s;
  if (pass == 0) {
    s.prefix = 0;
    s.need = D.seg_need;
    s.done = D.seg_need == 0;
    s.pad = 0;
    if (s.done) s.prefix = ~0ull;  // nothing is selected
  } else {
    s = state[bh];
  }
  __syncthreads();
  if (s.done) {
    if (pass == 0 && threadIdx.x == 0) state[bh] = s;
    return;
  }
  const unsigned* g = hist + (bh * kPasses + pass) * kBins;
  unsigned c[8];
  long long mine = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    c[i] = g[kBins - 1 - (threadIdx.x * 8 + i)];
    mine += c[i];
  }
  typedef cub::BlockScan<long long, 256> Scan;
  __shared__ typename Scan::TempStorage tmp;
  long long before;
  Scan(tmp).ExclusiveSum(mine, before);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (before < s.need && s.need <= before + (long long)c[i]) {
      const unsigned digit = kBins - 1 - (threadIdx.x * 8 + i);
      SelState o;
      o.prefix = s.prefix | ((unsigned long long)digit << c_shift[pass]);
      o.need = s.need - before;
      o.done = (o.need == (long long)c[i]) ? 1 : 0;
      o.pad = 0;
      state[bh] = o;
      if (!o.done && pass == kPasses - 1) lh_report(D.status, LH_ERR_DEVICE_BOUNDS, 100);
    }
    before += c[i];
  }
}

// Stratified selection: one block of 256 threads per (b, h) and chunk finds
// the chunk's m-th largest key by the same 11-bit radix passes, reading the
// chunk's keys once per pass (they stay in L1/L2) and counting digits in
// shared memory; it stops as soon as every key left in the chosen digit is
// needed.  state[bs].prefix is then the threshold: selected(f) <=> key(f) >=
// prefix, and exactly m keys of the chunk pass it (keys are unique).
__global__ void __launch_bounds__(256) k_sel_chunk(LhDims D, const float* __restrict__ qk,
                                                   const float* __restrict__ kq,
                                                   SelState* __restrict__ state) {
  const int64_t bs = blockIdx.x;                 // (b, h) x chunk
  const int64_t bh = bs / D.nseg;
  const int64_t s = bs - bh * D.nseg;
  const int64_t lo = s * D.n_cand / D.nseg;
  const int64_t hi_f = (s + 1) * D.n_cand / D.nseg;
  const float* q = qk + bh * D.P;
  const float* k = kq + bh * D.P;
  __shared__ unsigned h[kBins];
  __shared__ SelState sh;
  typedef cub::BlockScan<long long, 256> Scan;
  __shared__ typename Scan::TempStorage tmp;
  SelState st;
  st.prefix = 0;
  st.need = D.seg_need;
  st.done = 0;
  st.pad = 0;
  for (int pass = 0; pass < kPasses; ++pass) {
    for (int i = threadIdx.x; i < kBins; i += blockDim.x) h[i] = 0;
    __syncthreads();
    const int shift = c_shift[pass];
    const int hi = shift + c_width[pass];
    const unsigned mask = (1u << c_width[pass]) - 1u;
    for (int64_t f0 = lo; f0 < hi_f; f0 += blockDim.x) {
      const int64_t f = f0 + threadIdx.x;
      bool in = f < hi_f;
      unsigned digit = 0;
      if (in) {
        const unsigned long long key = entry_key(q, k, f);
        in = (hi >= 64) || ((key >> hi) == (st.prefix >> hi));
        digit = (unsigned)(key >> shift) & mask;
      }
      const unsigned act = __ballot_sync(0xffffffffu, in);
      if (in) {
        const unsigned peers = __match_any_sync(act, digit);
        if ((threadIdx.x & 31) == (unsigned)(__ffs(peers) - 1)) atomicAdd(&h[digit], __popc(peers));
      }
    }
    __syncthreads();
    unsigned c[8];
    long long mine = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      c[i] = h[kBins - 1 - (threadIdx.x * 8 + i)];
      mine += c[i];
    }
    long long before;
    Scan(tmp).ExclusiveSum(mine, before);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (before < st.need && st.need <= before + (long long)c[i]) {
        const unsigned digit = kBins - 1 - (threadIdx.x * 8 + i);
        SelState o;
        o.prefix = st.prefix | ((unsigned long long)digit << c_shift[pass]);
        o.need = st.need - before;
        o.done = (o.need == (long long)c[i]) ? 1 : 0;
        o.pad = 0;
        sh = o;
      }
      before += c[i];
    }
    __syncthreads();   // sh written by exactly one thread (need <= keys left)
    st = sh;
    __syncthreads();   // everyone has read sh and h before the next pass clears h
    if (st.done) break;
  }
  if (threadIdx.x == 0) {
    if (!st.done) lh_report(D.status, LH_ERR_DEVICE_BOUNDS, 103);
    state[bs] = st;
  }
}

// thr: the (b, h)'s segment states; an entry of level l < L-1 is compared with
// the threshold of its segment: segment 0 in mode 0, segment l in mode 1, and
// in mode 2 its chunk s, the one with floor(s C / n) <= f < floor((s+1) C / n),
// i.e. s = floor(((f+1) n - 1) / C).
__device__ __forceinline__ bool selected_entry(const LhDims& D, const float* q, const float* k,
                                               const SelState* thr, int l, int64_t f) {
  if (l == D.L - 1) return true;
  int64_t seg = 0;
  if (D.select_mode == 2) seg = ((f + 1) * D.nseg - 1) / D.n_cand;
  else if (D.nseg > 1) seg = l;
  return entry_key(q, k, f) >= thr[seg].prefix;
}

// Number of selected entries that end on token t.
__device__ __forceinline__ int count_at(const LhDims& D, const float* q, const float* k,
                                        const SelState* thr, int64_t t) {
  int n = 0;
  const uint32_t t1 = (uint32_t)(t + 1);  // N < 2^31
  for (int l = 0; l < D.L; ++l) {
    const uint32_t span = (uint32_t)D.lvl_span[l];
    if (t1 % span) break;  // spans are nested: no coarser level ends here either
    n += selected_entry(D, q, k, thr, l, D.lvl_off[l] + t1 / span - 1);
  }
  return n;
}

__global__ void __launch_bounds__(kOrderThreads) k_order_count(LhDims D, const float* __restrict__ qk,
                                                              const float* __restrict__ kq,
                                                              const SelState* __restrict__ state,
                                                              int* __restrict__ blk_cnt, int nblk) {
  const int64_t bh = blockIdx.y;
  const SelState* thr = state + bh * D.nseg;
  const float* q = qk + bh * D.P;
  const float* k = kq + bh * D.P;
  const int64_t t0 = (int64_t)blockIdx.x * kOrderTile;
  int n = 0;
  for (int i = 0; i < kOrderItems; ++i) {
    const int64_t t = t0 + (int64_t)i * kOrderThreads + threadIdx.x;
    if (t < D.N) n += count_at(D, q, k, thr, t);
  }
  typedef cub::BlockReduce<int, kOrderThreads> Red;
  __shared__ typename Red::TempStorage tmp;
  const int tot = Red(tmp).Sum(n);
  if (threadIdx.x == 0) blk_cnt[bh * nblk + blockIdx.x] = tot;
}

// One block per (b, h): exclusive scan of the block counts, in place.
__global__ void __launch_bounds__(1024) k_order_scan(LhDims D, int* __restrict__ blk_cnt, int nblk) {
  const int64_t bh = blockIdx.x;
  int* c = blk_cnt + bh * nblk;
  typedef cub::BlockScan<int, 1024> Scan;
  __shared__ typename Scan::TempStorage tmp;
  __shared__ int carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < nblk; base += 1024) {
    const int i = base + threadIdx.x;
    const int x = i < nblk ? c[i] : 0;
    int ex, agg;
    Scan(tmp).ExclusiveSum(x, ex, agg);
    if (i < nblk) c[i] = carry + ex;
    __syncthreads();
    if (threadIdx.x == 0) carry += agg;
    __syncthreads();
  }
  if (threadIdx.x == 0 && carry != D.S) lh_report(D.status, LH_ERR_DEVICE_BOUNDS, 101);
}

__global__ void __launch_bounds__(kOrderThreads) k_order_emit(LhDims D, const float* __restrict__ qk,
                                                             const float* __restrict__ kq,
                                                             const SelState* __restrict__ state,
                                                             const int* __restrict__ blk_off, int nblk,
                                                             int32_t* __restrict__ sel_idx,
                                                             int32_t* __restrict__ slot_map) {
  const int64_t bh = blockIdx.y;
  const SelState* thr = state + bh * D.nseg;
  const float* q = qk + bh * D.P;
  const float* k = kq + bh * D.P;
  // each thread owns kOrderItems consecutive tokens so the scan order is t order
  const int64_t t0 = (int64_t)blockIdx.x * kOrderTile + (int64_t)threadIdx.x * kOrderItems;
  int n = 0;
  for (int i = 0; i < kOrderItems; ++i) {
    const int64_t t = t0 + i;
    if (t < D.N) n += count_at(D, q, k, thr, t);
  }
  typedef cub::BlockScan<int, kOrderThreads> Scan;
  __shared__ typename Scan::TempStorage tmp;
  int ex;
  Scan(tmp).ExclusiveSum(n, ex);
  int slot = blk_off[bh * nblk + blockIdx.x] + ex;
  int32_t* si = sel_idx + bh * D.S;
  int32_t* sm = slot_map + bh * D.P;
  for (int i = 0; i < kOrderItems; ++i) {
    const int64_t t = t0 + i;
    if (t >= D.N) break;
    const uint32_t t1 = (uint32_t)(t + 1);
    for (int l = 0; l < D.L; ++l) {
      const uint32_t span = (uint32_t)D.lvl_span[l];
      if (t1 % span) break;
      const int64_t f = D.lvl_off[l] + t1 / span - 1;
      if (selected_entry(D, q, k, thr, l, f)) {
        if (slot < D.S) si[slot] = (int32_t)f;
        else lh_report(D.status, LH_ERR_DEVICE_BOUNDS, 102);
        sm[f] = slot++;
      } else {
        sm[f] = -1;
      }
    }
  }
}

inline int64_t order_blocks(const LhDims& D) { return (D.N + kOrderTile - 1) / kOrderTile; }

}  // namespace

size_t lh_select_ws_bytes(const LhDims& D) {
  const int64_t BH = (int64_t)D.B * D.H;
  const int64_t BS = BH * D.nseg;
  size_t b = 0;
  if (D.select_mode != 2) b += (size_t)BS * kPasses * kBins * sizeof(unsigned);  // histograms
  b += (size_t)BS * sizeof(SelState);
  b = (b + 255) & ~(size_t)255;
  b += (size_t)BH * order_blocks(D) * sizeof(int);
  return (b + 255) & ~(size_t)255;
}

cudaError_t lh_launch_select(const LhDims& D, const float* qk, const float* kq,
                             int32_t* sel_idx, int32_t* slot_map, void* ws, cudaStream_t st,
                             int* launches) {
  const int64_t BH = (int64_t)D.B * D.H;
  const int64_t BS = BH * D.nseg;                 // (b, h) x selection segment
  const size_t hist_bytes =
      D.select_mode == 2 ? 0 : (size_t)BS * kPasses * kBins * sizeof(unsigned);
  unsigned* hist = reinterpret_cast<unsigned*>(ws);
  SelState* state = reinterpret_cast<SelState*>(reinterpret_cast<char*>(ws) + hist_bytes);
  size_t off = hist_bytes + (size_t)BS * sizeof(SelState);
  off = (off + 255) & ~(size_t)255;
  int* blk = reinterpret_cast<int*>(reinterpret_cast<char*>(ws) + off);
  const int nblk = (int)order_blocks(D);
  int n = 0;
  if (D.select_mode == 2) {
    k_sel_chunk<<<(unsigned)BS, 256, 0, st>>>(D, qk, kq, state);
    n += 1;
  } else if (D.n_cand > 0) {
    cudaError_t e = cudaMemsetAsync(hist, 0, hist_bytes, st);
    if (e != cudaSuccess) return e;
    // ~8 candidates per thread per block keeps every SM busy on one head too
    int64_t per = (D.seg_len[0] + 148 * 4 - 1) / (148 * 4);   // segment 0 is the largest
    per = per < 2048 ? 2048 : per;
    const unsigned gx = (unsigned)((D.seg_len[0] + per - 1) / per);
    for (int pass = 0; pass < kPasses; ++pass) {
      k_sel_hist<<<dim3(gx, (unsigned)BS), 256, 0, st>>>(D, qk, kq, hist, state, pass);
      k_sel_find<<<(unsigned)BS, 256, 0, st>>>(D, hist, state, pass);
      n += 2;
    }
  } else {
    k_sel_find<<<(unsigned)BS, 256, 0, st>>>(D, hist, state, 0);   // reads no histogram
    n += 1;
  }
  k_order_count<<<dim3(nblk, (unsigned)BH), kOrderThreads, 0, st>>>(D, qk, kq, state, blk, nblk);
  k_order_scan<<<(unsigned)BH, 1024, 0, st>>>(D, blk, nblk);
  k_order_emit<<<dim3(nblk, (unsigned)BH), kOrderThreads, 0, st>>>(D, qk, kq, state, blk, nblk,
                                                                   sel_idx, slot_map);
  n += 3;
  if (launches) *launches = n;
  return cudaGetLastError();
}
