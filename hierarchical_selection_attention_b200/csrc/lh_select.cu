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
// t; the emit pass writes sel_idx (slot -> entry) and slot_map (entry ->
// slot or -1).
//
// One launch does all of it.  Each (b, h) gets one thread-block cluster of
// kCl CTAs; CTA c owns a contiguous range of base tokens (a multiple of
// p^(L-1) long) and, at every level, the entries that end inside it.
//  Selection (modes 0, 1): per radix pass every CTA counts the digits of
//   its own keys in shared memory; after a cluster barrier the leader CTA
//   sums the kCl histograms through distributed shared memory, picks the
//   digit and publishes the new state; after a second barrier every CTA
//   reads it.  Keys are re-read from global memory each pass (they stay in
//   L2).  Mode 2: the cluster's CTAs share out the head's chunks, each chunk
//   selected by one CTA with a shared-memory histogram.
//  Order: every CTA marks which of its entries are selected in shared-memory
//   bit masks (level by level, for a window of at most kWin tokens at a
//   time), counts them, takes its first slot from the counts of the
//   lower-ranked CTAs (read through distributed shared memory) and emits its
//   tokens in order from the masks.
// The cluster barriers are hardware barriers that every thread of every CTA
// reaches (all control flow around them is uniform across the cluster), so
// nothing spins on memory.  Integer work only: the result is bit-exact and
// the same on every run.
#include <cooperative_groups.h>
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

constexpr int kSelThreads = 512;
constexpr int kWarps = kSelThreads / 32;
constexpr int kBinsPer = kBins / kSelThreads;         // digits per thread in a find step
constexpr int kUnroll = 8;                            // keys in flight per thread
constexpr int kItems = 4;                             // tokens per thread per emit tile
constexpr int kTile = kSelThreads * kItems;
constexpr int64_t kWin = 65536;                       // tokens per selection-mask window
constexpr int kMaskWords = (int)(2 * kWin / 32);      // all levels of a window (p >= 2)

namespace cg = cooperative_groups;

__device__ __forceinline__ unsigned long long entry_key(const float* qk, const float* kq,
                                                        int64_t f) {
  const float r = fmaxf(__ldg(qk + f), __ldg(kq + f));
  return ((unsigned long long)__float_as_uint(r) << 32) |
         (unsigned long long)(0xffffffffu - (uint32_t)f);
}

typedef cub::BlockScan<long long, kSelThreads> ScanLL;
typedef cub::BlockScan<int, kSelThreads> ScanI;
typedef cub::BlockReduce<long long, kSelThreads> RedLL;

struct SelSmem {
  unsigned hist[kBins];
  unsigned red[kBins];         // this CTA's slice of the cluster-summed histogram
  uint32_t mask[kMaskWords];   // selection bits of a window, level after level
  SelState st;                 // the leader's current state (read by the cluster)
  long long cnt;               // this CTA's selected-entry count
  long long base;              // its first slot
  union {
    typename ScanLL::TempStorage scan_ll;
    typename ScanI::TempStorage scan_i;
    typename RedLL::TempStorage red_ll;
  } tmp;
};

// Add the digits of the keys f in [lo, hi) that match `prefix` above this
// pass's digit to h (warp-aggregated shared-memory atomics).  Called by the
// whole block; every thread runs the same rounds.  kUnroll keys per thread
// are loaded before any is counted, so their loads overlap.
__device__ __forceinline__ void count_digits(const float* q, const float* k, int64_t lo,
                                             int64_t hi, unsigned long long prefix, int pass,
                                             unsigned* h) {
  const int shift = c_shift[pass];
  const int top = shift + c_width[pass];
  const unsigned mask = (1u << c_width[pass]) - 1u;
  const int64_t span = hi > lo ? hi - lo : 0;
  const int64_t per = (int64_t)blockDim.x * kUnroll;
  for (int64_t r0 = 0; r0 < span; r0 += per) {
    unsigned long long key[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t f = lo + r0 + (int64_t)u * blockDim.x + threadIdx.x;
      key[u] = f < hi ? entry_key(q, k, f) : 0ull;
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t f = lo + r0 + (int64_t)u * blockDim.x + threadIdx.x;
      const bool in = f < hi && ((top >= 64) || ((key[u] >> top) == (prefix >> top)));
      const unsigned digit = (unsigned)(key[u] >> shift) & mask;
      const unsigned act = __ballot_sync(0xffffffffu, in);
      if (in) {
        const unsigned peers = __match_any_sync(act, digit);
        if ((threadIdx.x & 31) == (unsigned)(__ffs(peers) - 1)) atomicAdd(&h[digit], __popc(peers));
      }
    }
  }
}

// The digit of this pass that holds the need-th largest key, from the
// per-digit counts count(d) (thread t owns digits 2047 - kBinsPer t
// downwards).  The new state goes to *out, written by the one thread whose
// digit it is.  Whole block.
template <typename Count>
__device__ __forceinline__ void find_digit(const SelState& s, int pass, Count count,
                                           SelState* out, typename ScanLL::TempStorage& tmp) {
  unsigned c[kBinsPer];
  long long mine = 0;
#pragma unroll
  for (int i = 0; i < kBinsPer; ++i) {
    c[i] = count(kBins - 1 - (threadIdx.x * kBinsPer + i));
    mine += c[i];
  }
  long long before;
  ScanLL(tmp).ExclusiveSum(mine, before);
#pragma unroll
  for (int i = 0; i < kBinsPer; ++i) {
    if (before < s.need && s.need <= before + (long long)c[i]) {
      const unsigned digit = kBins - 1 - (threadIdx.x * kBinsPer + i);
      SelState o;
      o.prefix = s.prefix | ((unsigned long long)digit << c_shift[pass]);
      o.need = s.need - before;
      o.done = (o.need == (long long)c[i]) ? 1 : 0;
      o.pad = 0;
      *out = o;
    }
    before += c[i];
  }
}

__device__ __forceinline__ SelState start_state(int64_t need) {
  SelState s;
  s.prefix = 0;
  s.need = need;
  s.done = need == 0;
  s.pad = 0;
  if (s.done) s.prefix = ~0ull;   // nothing is selected
  return s;
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
  return entry_key(q, k, f) >= __ldcg(&thr[seg].prefix);
}

// Selection bits of the entries that end in tokens [w0, w1) (multiples of
// the coarsest span), level after level: level l's entries
// [w0 / p^l, w1 / p^l) at bit offsets moff[l] + j.  Returns this thread's
// count of set bits.  Whole block; warps take 32-entry words, kUnroll/2
// words in flight.
__device__ __forceinline__ int build_masks(const LhDims& D, const float* q, const float* k,
                                           const SelState* thr, int64_t w0, int64_t w1,
                                           uint32_t* mask, const int* moff) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int W = kUnroll / 2;
  int n = 0;
  for (int l = 0; l < D.L; ++l) {
    const int64_t sp = D.lvl_span[l];
    const int64_t e0 = w0 / sp, ne = (w1 - w0) / sp;
    const int words = (int)((ne + 31) / 32);
    uint32_t* m = mask + moff[l] / 32;
    for (int wb = warp * W; wb < words; wb += kWarps * W) {
      bool sel[W];
#pragma unroll
      for (int u = 0; u < W; ++u) {
        const int64_t j = (int64_t)(wb + u) * 32 + lane;
        sel[u] = (wb + u) < words && j < ne &&
                 selected_entry(D, q, k, thr, l, D.lvl_off[l] + e0 + j);
      }
#pragma unroll
      for (int u = 0; u < W; ++u) {
        const uint32_t b = __ballot_sync(0xffffffffu, sel[u]);
        if (lane == 0 && wb + u < words) {
          m[wb + u] = b;
          n += __popc(b);
        }
      }
    }
  }
  return n;
}

__device__ __forceinline__ bool mask_bit(const uint32_t* mask, int64_t bit) {
  return (mask[bit >> 5] >> (bit & 31)) & 1u;
}

// One cluster of CL CTAs per (b, h) (blockIdx.y); see the file comment.
template <int CL>
__global__ void __launch_bounds__(kSelThreads) k_select(LhDims D, const float* __restrict__ qk,
                                                        const float* __restrict__ kq,
                                                        SelState* __restrict__ state,
                                                        int32_t* __restrict__ sel_idx,
                                                        int32_t* __restrict__ slot_map) {
  cg::cluster_group cluster = cg::this_cluster();
  __shared__ SelSmem sm;
  const int c = (int)cluster.block_rank();
  const int64_t bh = blockIdx.y;
  const float* q = qk + bh * D.P;
  const float* k = kq + bh * D.P;
  SelState* thr = state + bh * D.nseg;
  // this CTA's tokens [t0, t1): whole coarsest-level windows
  const int64_t span_top = D.lvl_span[D.L - 1];
  const int64_t n_top = D.lvl_size[D.L - 1];
  const int64_t tc = (n_top + CL - 1) / CL * span_top;
  const int64_t t0 = min((int64_t)c * tc, D.N), t1 = min(t0 + tc, D.N);

  // ---- selection
  if (D.select_mode == 2) {
    // chunks s = c, c + CL, ...: one CTA runs all radix passes of a chunk
    for (int64_t sg = c; sg < D.nseg; sg += CL) {
      const int64_t lo = sg * D.n_cand / D.nseg, hi = (sg + 1) * D.n_cand / D.nseg;
      SelState st = start_state(D.seg_need);
      for (int pass = 0; pass < kPasses && !st.done; ++pass) {
        for (int i = threadIdx.x; i < kBins; i += blockDim.x) sm.hist[i] = 0;
        __syncthreads();
        count_digits(q, k, lo, hi, st.prefix, pass, sm.hist);
        __syncthreads();
        find_digit(st, pass, [&](int d) { return sm.hist[d]; }, &sm.st, sm.tmp.scan_ll);
        __syncthreads();                // sm.st written by exactly one thread
        st = sm.st;
        __syncthreads();                // read before the next pass clears hist
      }
      if (threadIdx.x == 0) {
        if (!st.done) lh_report(D.status, LH_ERR_DEVICE_BOUNDS, 103);
        thr[sg] = st;
      }
    }
  } else {
    constexpr int kSlice = kBins / CL;  // digits whose cluster sum this CTA forms
    for (int sg = 0; sg < D.nseg; ++sg) {
      // levels of this segment: all finer ones (mode 0) or level sg (mode 1)
      const int l_lo = D.nseg > 1 ? sg : 0;
      const int l_hi = D.nseg > 1 ? sg + 1 : D.L - 1;
      SelState st = start_state(D.seg_need);
      for (int pass = 0; pass < kPasses && !st.done; ++pass) {
        for (int i = threadIdx.x; i < kBins; i += blockDim.x) sm.hist[i] = 0;
        __syncthreads();
        for (int l = l_lo; l < l_hi; ++l) {
          const int64_t sp = D.lvl_span[l];
          count_digits(q, k, D.lvl_off[l] + t0 / sp, D.lvl_off[l] + t1 / sp, st.prefix, pass,
                       sm.hist);
        }
        cluster.sync();                 // every CTA's histogram is complete
        for (int i = threadIdx.x; i < kSlice; i += blockDim.x) {
          unsigned tot = 0;
#pragma unroll
          for (int r = 0; r < CL; ++r) tot += cluster.map_shared_rank(sm.hist, r)[c * kSlice + i];
          sm.red[i] = tot;
        }
        cluster.sync();                 // the summed histogram lies in the CTAs' slices
        if (c == 0)
          find_digit(st, pass, [&](int d) {
            return cluster.map_shared_rank(sm.red, d / kSlice)[d % kSlice];
          }, &sm.st, sm.tmp.scan_ll);
        cluster.sync();                 // the leader's state is published
        st = *cluster.map_shared_rank(&sm.st, 0);
      }
      if (c == 0 && threadIdx.x == 0) {
        if (!st.done) lh_report(D.status, LH_ERR_DEVICE_BOUNDS, 100);
        thr[sg] = st;
      }
      cluster.sync();                   // every CTA has read the leader's sm.st
    }
  }
  __threadfence();
  cluster.sync();                       // thresholds in global memory, seen by the cluster

  // ---- order.  Bit offsets of each level inside a window's masks.
  __shared__ int moff[LH_MAX_LEVELS];
  if (threadIdx.x == 0) {
    int o = 0;
    for (int l = 0; l < D.L; ++l) {
      moff[l] = o;
      o += (int)(((kWin / D.lvl_span[l]) + 31) / 32) * 32;
    }
  }
  __syncthreads();
  const int64_t win = kWin / span_top * span_top;    // a multiple of the coarsest span
  const int64_t nwin = (t1 - t0 + win - 1) / win;
  long long n = 0;
  for (int64_t w0 = t0; w0 < t1; w0 += win) {
    n += build_masks(D, q, k, thr, w0, min(w0 + win, t1), sm.mask, moff);
    __syncthreads();                    // masks rebuilt by the next window
  }
  n = RedLL(sm.tmp.red_ll).Sum(n);
  if (threadIdx.x == 0) sm.cnt = n;
  cluster.sync();
  if (threadIdx.x == 0) {
    long long base = 0, total = 0;
    for (int r = 0; r < CL; ++r) {
      const long long x = *cluster.map_shared_rank(&sm.cnt, r);
      if (r < c) base += x;
      total += x;
    }
    sm.base = base;
    if (c == 0 && total != D.S) lh_report(D.status, LH_ERR_DEVICE_BOUNDS, 101);
  }
  __syncthreads();
  int32_t* si = sel_idx + bh * D.S;
  int32_t* smap = slot_map + bh * D.P;
  long long slot0 = sm.base;
  for (int64_t w0 = t0; w0 < t1; w0 += win) {
    const int64_t w1 = min(w0 + win, t1);
    if (nwin > 1) {                     // one window: its masks are still there
      build_masks(D, q, k, thr, w0, w1, sm.mask, moff);
      __syncthreads();
    }
    for (int64_t tt = w0; tt < w1; tt += kTile) {
      const int64_t ta = tt + (int64_t)threadIdx.x * kItems;   // kItems consecutive tokens
      int cnt = 0;
#pragma unroll
      for (int u = 0; u < kItems; ++u) {
        const int64_t t = ta + u;
        if (t >= w1) break;
        const int64_t t1p = t + 1;
        for (int l = 0; l < D.L; ++l) {
          const int64_t sp = D.lvl_span[l];
          if (t1p % sp) break;
          cnt += mask_bit(sm.mask, moff[l] + (t1p / sp - 1 - w0 / sp));
        }
      }
      int ex, agg;
      ScanI(sm.tmp.scan_i).ExclusiveSum(cnt, ex, agg);
      long long slot = slot0 + ex;
      for (int u = 0; u < kItems; ++u) {
        const int64_t t = ta + u;
        if (t >= w1) break;
        const int64_t t1p = t + 1;
        for (int l = 0; l < D.L; ++l) {
          const int64_t sp = D.lvl_span[l];
          if (t1p % sp) break;
          const int64_t i = t1p / sp - 1;
          const int64_t f = D.lvl_off[l] + i;
          if (mask_bit(sm.mask, moff[l] + (i - w0 / sp))) {
            if (slot < D.S) si[slot] = (int32_t)f;
            else lh_report(D.status, LH_ERR_DEVICE_BOUNDS, 102);
            smap[f] = (int32_t)slot++;
          } else {
            smap[f] = -1;
          }
        }
      }
      slot0 += agg;
      __syncthreads();                  // scan storage reused by the next tile
    }
  }
  cluster.sync();                       // no CTA leaves while others read its shared memory
}

template <int CL>
cudaError_t launch_select(const LhDims& D, const float* qk, const float* kq, SelState* state,
                          int32_t* sel_idx, int32_t* slot_map, cudaStream_t st) {
  if (CL > 8) {
    const cudaError_t e =
        cudaFuncSetAttribute(k_select<CL>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(CL, (unsigned)((int64_t)D.B * D.H));
  cfg.blockDim = dim3(kSelThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_select<CL>, D, qk, kq, state, sel_idx, slot_map);
}

}  // namespace

size_t lh_select_ws_bytes(const LhDims& D) {
  const int64_t BS = (int64_t)D.B * D.H * D.nseg;
  return ((size_t)BS * sizeof(SelState) + 255) & ~(size_t)255;   // per-segment thresholds
}

cudaError_t lh_launch_select(const LhDims& D, const float* qk, const float* kq,
                             int32_t* sel_idx, int32_t* slot_map, void* ws, cudaStream_t st,
                             int* launches) {
  SelState* state = reinterpret_cast<SelState*>(ws);
  // 16-CTA clusters where the device schedules them, else the portable 8
  cudaError_t e = launch_select<16>(D, qk, kq, state, sel_idx, slot_map, st);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    e = launch_select<8>(D, qk, kq, state, sel_idx, slot_map, st);
  }
  if (launches) *launches = 1;
  return e != cudaSuccess ? e : cudaGetLastError();
}
