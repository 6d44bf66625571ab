// Stage kernel 1 of the MicroAdam step ([MicroAdam ¶1] = paragraph 1 of
// "MicroAdam (Sparse-Gradient Adaptive Optimization with Quantized Error
// Feedback)"), one CTA per block of B_d parameters:
//   a_t = g_t + Q^{-1}(e_t, delta_t, Delta_t)      (in registers, never stored)
//   (I_t, V_t) = Top-k of |a_t| (ties to the lower index), written in
//   ascending index order to row t mod m of the window G,
//   the residual (a_t with the selected entries zeroed) reduced to its block
//   min/max and folded into the global (-delta_{t+1}, Delta_{t+1}) pair with
//   one pair of integer atomics per CTA,
//   and, for the blocks assigned to this kernel (j & 7 < update_split), the
//   AdamStats update of the block's parameters (block_update), which needs the
//   new row but not delta_{t+1}; that moves HBM traffic into this
//   arithmetic-heavier kernel.
//
// Exact Top-k in two tiers:
//  * candidate tier: a lower bound tau_lo for the k-th largest magnitude is
//    estimated from one sample per thread (a high order statistic of the warps'
//    top-2 samples, aiming at a few times k candidates); elements with
//    |a| >= tau_lo are written, in index order, to a shared-memory list; an
//    exact radix select on the list uses digits that start at the highest bit
//    where tau_lo and the block's largest magnitude differ, so keys clustered
//    in a narrow range (the usual case once the error feedback carries
//    quantization noise) still spread over the histogram. One pass usually
//    isolates the k-th key; the whole tier takes about ten block barriers;
//  * full tier, when the estimate fails (fewer than k or more than the list
//    capacity): the same exact radix select on all keys, re-reading the block
//    from L2 on every pass.
// Both tiers produce identical results: the k largest keys, ties to the lower
// index. HBM traffic per parameter: 2 B gradient + 0.5 B codes read; per
// selected entry 4 B written; plus block_update's traffic for its blocks.
#include <algorithm>

#include "mua_kernels.cuh"

namespace mua {
namespace {

// Digit bin holding the krem-th largest remaining key: the largest b with
// (count of bins >= b) >= krem. Writes the bin and the count strictly above it
// to s_res[0], s_res[1].
template <int T>
__device__ __forceinline__ void find_bin(const uint32_t* hist, int nbins, int krem,
                                         uint32_t* scan_scratch, uint32_t* s_res) {
  const int tid = threadIdx.x;
  const int per = (nbins >= T) ? nbins / T : 1;
  const int active = nbins / per;
  uint32_t own = 0;
  if (tid < active) {
    for (int b = 0; b < per; ++b) own += hist[tid * per + b];
  }
  uint32_t total;
  const uint32_t incl = block_inclusive_scan<T, uint32_t>(own, scan_scratch, total);
  if (tid < active) {
    uint32_t running = total - incl;  // keys in bins above this thread's range
    for (int b = per - 1; b >= 0; --b) {
      const uint32_t h = hist[tid * per + b];
      if (running < (uint32_t)krem && running + h >= (uint32_t)krem) {
        s_res[0] = (uint32_t)(tid * per + b);
        s_res[1] = running;
      }
      running += h;
    }
  }
}

struct SelectShared {
  uint32_t scan32[32];
  uint32_t scan32b[32];
  uint32_t wsum[32];
  uint32_t wmax[32];
  unsigned long long scan64[32];
  unsigned long long gkey[32];
  uint32_t gcnt;
  uint32_t mm[2];     // block residual (-min, max) bit patterns
  uint32_t arrived;   // warps that have folded their min/max
  uint32_t res[3];
  uint32_t top[64];
  uint32_t tau_lo;
  float mn[32], mx[32];
  float levels[16];
  float w1[kMaxWindow], w2[kMaxWindow];
};

// Writes a selected entry to its row slot.
__device__ __forceinline__ void put_entry(uint32_t* row, uint32_t pos, int k, uint32_t idx,
                                          uint32_t abits) {
  if (pos < (uint32_t)k) {
    const uint32_t vb = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(abits)));
    row[pos] = (idx & 0xFFFFu) | (vb << 16);
  }
}

// a_t of the 8 elements of chunk c of thread tid, re-read from global memory
// (the block was just streamed, so this hits L2). Elements past L are +0.
template <int T, bool VEC>
__device__ __forceinline__ void chunk_values(const uint16_t* grads, const uint8_t* codes,
                                             int64_t start, int L, int c, const float* lv,
                                             uint32_t (&ab)[kChunk]) {
  uint4 gv;
  uint32_t cv;
  const int tid = threadIdx.x;
  const int e0 = elem_index<T>(c, tid, 0);
  if (VEC && e0 + kChunk <= L) {
    gv = *reinterpret_cast<const uint4*>(grads + start + e0);
    cv = *reinterpret_cast<const uint32_t*>(codes + ((start + e0) >> 1));
  } else {
    uint32_t w[4] = {0u, 0u, 0u, 0u};
    uint32_t cw = 0u;
    for (int e = 0; e < kChunk; ++e) {
      if (e0 + e < L) {
        const int64_t i = start + e0 + e;
        const uint32_t byte = codes[i >> 1];
        w[e >> 1] |= (uint32_t)grads[i] << (16 * (e & 1));
        cw |= ((i & 1) ? (byte >> 4) : (byte & 0xFu)) << (4 * e);
      }
    }
    gv = make_uint4(w[0], w[1], w[2], w[3]);
    cv = cw;
  }
#pragma unroll
  for (int e = 0; e < kChunk; ++e) {
    const float a = __fadd_rn(__uint_as_float(grad_bits(gv, e)), lv[(cv >> (4 * e)) & 0xFu]);
    ab[e] = (e0 + e < L) ? __float_as_uint(a) : 0u;
  }
}

// Exact radix select over every key of the block (full tier, used when the
// candidate estimate fails): digits of 11, 11 and 9 bits, each pass re-reading
// the block from L2. Writes the row and folds every non-selected value into
// rmin/rmax.
// The arguments are plain pointers and values: a reference to the kernel's
// parameter block would make every CTA copy that block to local memory.
template <int T, bool VEC>
__device__ __noinline__ void select_full(const uint16_t* grads, const uint8_t* codes,
                                         uint32_t* hdr, int64_t start, int L, int k,
                                         const float* lv, uint32_t* hist, SelectShared& sh,
                                         uint32_t* row, float& rmin, float& rmax) {
  const int tid = threadIdx.x;
  uint32_t prefix = 0u, pmask = 0u;
  int krem = k;
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 20 : (pass == 1 ? 9 : 0);
    const int nbins = pass == 2 ? 512 : kHistBins;
    for (int b = tid; b < nbins; b += T) hist[b] = 0u;
    if (tid == 0) sh.res[0] = sh.res[1] = 0u;
    __syncthreads();
    for (int c = 0; c < kChunks; ++c) {
      uint32_t ab[kChunk];
      chunk_values<T, VEC>(grads, codes, start, L, c, lv, ab);
#pragma unroll
      for (int e = 0; e < kChunk; ++e)  // digits lie in bits 0..30
        if ((ab[e] & pmask) == prefix) atomicAdd(&hist[(ab[e] >> shift) & (nbins - 1)], 1u);
    }
    __syncthreads();
    if (pass == 0 && tid == 0) {
      uint32_t bad = 0;  // keys >= 0x7F800000 (bins 0x7F8..) are +-inf or NaN
      for (int b = 0x7F8; b < kHistBins; ++b) bad |= hist[b];
      if (bad) atomicOr(&hdr[kHdrStatus], kStatusNonFinite);
    }
    find_bin<T>(hist, nbins, krem, sh.scan32, sh.res);
    __syncthreads();
    prefix |= sh.res[0] << shift;
    pmask |= (uint32_t)(nbins - 1) << shift;
    krem -= (int)sh.res[1];
    __syncthreads();
  }
  const uint32_t tau = prefix;
  const int need = krem;

  // Counts per chunk of keys > tau and == tau, packed: 16-bit field c holds
  // chunk c (each total <= 8T <= 8192).
  unsigned long long pg = 0ull, pe = 0ull;
  for (int c = 0; c < kChunks; ++c) {
    uint32_t ab[kChunk];
    chunk_values<T, VEC>(grads, codes, start, L, c, lv, ab);
    uint32_t ng = 0, ne = 0;
#pragma unroll
    for (int e = 0; e < kChunk; ++e) {
      const uint32_t key = ab[e] & 0x7FFFFFFFu;
      ng += key > tau;
      ne += key == tau;
    }
    pg |= (unsigned long long)ng << (16 * c);
    pe |= (unsigned long long)ne << (16 * c);
  }
  unsigned long long tg, te;
  const unsigned long long xg = block_inclusive_scan<T, unsigned long long>(pg, sh.scan64, tg) - pg;
  const unsigned long long xe = block_inclusive_scan<T, unsigned long long>(pe, sh.scan64, te) - pe;
  uint32_t base_g = 0, base_e = 0;
  for (int c = 0; c < kChunks; ++c) {
    uint32_t run_g = base_g + (uint32_t)((xg >> (16 * c)) & 0xFFFFu);
    uint32_t run_e = base_e + (uint32_t)((xe >> (16 * c)) & 0xFFFFu);
    base_g += (uint32_t)((tg >> (16 * c)) & 0xFFFFu);
    base_e += (uint32_t)((te >> (16 * c)) & 0xFFFFu);
    uint32_t ab[kChunk];
    chunk_values<T, VEC>(grads, codes, start, L, c, lv, ab);
#pragma unroll
    for (int e = 0; e < kChunk; ++e) {
      const uint32_t bits = ab[e];
      const uint32_t key = bits & 0x7FFFFFFFu;
      if (key > tau) {
        put_entry(row, run_g + min(run_e, (uint32_t)need), k, elem_index<T>(c, tid, e), bits);
        ++run_g;
      } else if (key == tau && run_e < (uint32_t)need) {
        put_entry(row, run_g + run_e, k, elem_index<T>(c, tid, e), bits);
        ++run_e;
      } else {
        if (key == tau) ++run_e;
        const float v = __uint_as_float(bits);
        rmin = fminf(rmin, v);
        rmax = fmaxf(rmax, v);
      }
    }
  }
}

// Exact radix select over the n-entry candidate list (index order); all keys lie
// in [tau_lo, kmax]. hist (>= 2048 words) must be zero on entry. Writes the
// row and folds the non-selected candidates into rmin/rmax.
template <int T>
__device__ void select_list(const uint32_t* cab, const uint16_t* cidx, int n, int k,
                            uint32_t tau_lo, uint32_t kmax, uint32_t* hist, SelectShared& sh,
                            uint32_t* row, float& rmin, float& rmax) {
  constexpr int NW = T / 32;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int q = (n + T - 1) / T;  // entries per thread, contiguous
  const int i0 = min(n, tid * q), i1 = min(n, i0 + q);

  // mode 0: selected = key >= thr; mode 1: key > thr, or key == thr for the
  // `need` lowest indices.
  uint32_t thr = tau_lo;
  int mode = 1, need = k;
  const uint32_t diff = kmax ^ tau_lo;
  if (diff != 0u) {
    int hi = 31 - __clz(diff);  // highest bit where candidates can differ
    uint32_t pmask = (hi >= 30) ? 0u : ((0xFFFFFFFFu << (hi + 1)) & 0x7FFFFFFFu);
    uint32_t prefix = tau_lo & pmask;
    int krem = k;
    bool first = true;
    while (hi >= 0) {
      const int width = min(11, hi + 1);
      const int shift = hi + 1 - width;
      const int nbins = 1 << width;
      if (!first) {
        for (int b = tid; b < nbins; b += T) hist[b] = 0u;
        __syncthreads();
      }
      first = false;
      for (int i = i0; i < i1; ++i) {
        const uint32_t key = cab[i] & 0x7FFFFFFFu;
        if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & (nbins - 1)], 1u);
      }
      __syncthreads();
      // Warp w owns bins [w*per, (w+1)*per); lane l owns per/32 of them.
      const int per = max(32, nbins / NW);
      const int per_lane = per / 32;
      const int b0 = wid * per + lane * per_lane;
      uint32_t own = 0;
      for (int b = 0; b < per_lane; ++b)
        if (b0 + b < nbins) own += hist[b0 + b];
      uint32_t incl = own;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += y;
      }
      if (lane == 31) sh.wsum[wid] = incl;
      __syncthreads();
      uint32_t above = 0;  // keys in the bins of the warps above this one
      for (int w = wid + 1; w < NW; ++w) above += sh.wsum[w];
      uint32_t running = above + (__shfl_sync(0xFFFFFFFFu, incl, 31) - incl);
      for (int b = per_lane - 1; b >= 0; --b) {
        if (b0 + b >= nbins) continue;
        const uint32_t h = hist[b0 + b];
        if (running < (uint32_t)krem && running + h >= (uint32_t)krem) {
          sh.res[0] = (uint32_t)(b0 + b);
          sh.res[1] = running;
          sh.res[2] = h;
        }
        running += h;
      }
      __syncthreads();
      const uint32_t bin = sh.res[0], abv = sh.res[1], inbin = sh.res[2];
      prefix |= bin << shift;
      pmask |= (uint32_t)(nbins - 1) << shift;
      krem -= (int)abv;
      hi = shift - 1;
      if (inbin == (uint32_t)krem) {  // the whole bin is selected: exact threshold
        thr = prefix;
        mode = 0;
        break;
      }
      __syncthreads();  // before the next pass clears the histogram
    }
    if (mode == 1) {
      thr = prefix;
      need = krem;
    }
  }

  // Positions in index order: counts of (key > thr, key == thr) per thread.
  uint32_t cg = 0, ce = 0;
  for (int i = i0; i < i1; ++i) {
    const uint32_t key = cab[i] & 0x7FFFFFFFu;
    if (mode == 0) {
      cg += key >= thr;
    } else {
      cg += key > thr;
      ce += key == thr;
    }
  }
  uint32_t tot;
  const uint32_t packed = cg | (ce << 16);  // n <= kCandCap < 2^16
  const uint32_t x = block_scan_1bar<T, uint32_t>(packed, sh.scan32b, tot) - packed;
  uint32_t run_g = x & 0xFFFFu, run_e = x >> 16;
  for (int i = i0; i < i1; ++i) {
    const uint32_t bits = cab[i];
    const uint32_t key = bits & 0x7FFFFFFFu;
    const bool gt = (mode == 0) ? key >= thr : key > thr;
    if (gt) {
      put_entry(row, run_g + min(run_e, (uint32_t)need), k, cidx[i], bits);
      ++run_g;
    } else if (mode == 1 && key == thr && run_e < (uint32_t)need) {
      put_entry(row, run_g + run_e, k, cidx[i], bits);
      ++run_e;
    } else {
      if (mode == 1 && key == thr) ++run_e;
      const float v = __uint_as_float(bits);
      rmin = fminf(rmin, v);
      rmax = fmaxf(rmax, v);
    }
  }
}

// Folds a residual min/max over the whole CTA into the global pair without a
// block barrier: every warp folds its partial into two shared words with
// atomics (both values are >= +0 as -min and max, so their bit patterns order
// like the values), and the last warp to arrive publishes them with one pair
// of global atomics. sh.mm[] and sh.arrived must be zero on entry; the caller
// resets them after a later barrier.
template <int T>
__device__ __forceinline__ void block_minmax_to_global(float rmin, float rmax, SelectShared& sh,
                                                       uint32_t* hdr, int pair_next) {
  constexpr int NW = T / 32;
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    rmin = fminf(rmin, __shfl_xor_sync(0xFFFFFFFFu, rmin, o));
    rmax = fmaxf(rmax, __shfl_xor_sync(0xFFFFFFFFu, rmax, o));
  }
  if (lane == 0) {
    atomicMax(&sh.mm[0], __float_as_uint(0.0f - rmin));  // canonical +0
    atomicMax(&sh.mm[1], __float_as_uint(rmax + 0.0f));
    __threadfence_block();
    if (atomicAdd(&sh.arrived, 1u) == NW - 1) {  // last warp: all partials are in
      __threadfence_block();
      atomicMax(&hdr[pair_next], atomicOr(&sh.mm[0], 0u));
      atomicMax(&hdr[pair_next + 1], atomicOr(&sh.mm[1], 0u));
    }
  }
}

// Everything after the loads for block j: gv/cv hold the thread's 4 chunks;
// sh.levels and sh.w1/w2 are filled; `work` is the dynamic shared-memory
// scratch (histogram + candidate list, then block_update). Ends with the
// block fully processed; the caller synchronizes before reusing `work`.
template <int T, bool VEC>
__device__ __forceinline__ void select_block(const StepArgs& A, int j,
                                             const uint4 (&gv)[kChunks],
                                             const uint32_t (&cv)[kChunks], uint8_t* work,
                                             SelectShared& sh) {
  uint32_t* hist = reinterpret_cast<uint32_t*>(work);
  uint32_t* cab = hist + kHistBins;
  uint16_t* cidx = reinterpret_cast<uint16_t*>(cab + kCandCap);

  const int tid = threadIdx.x;
  const int lane = tid & 31, wid = tid >> 5;
  constexpr int NW = T / 32;
  const Geometry& G = A.g;
  int64_t start;
  int L;
  block_span(A, j, start, L);
  const int k = (int)(((int64_t)L * G.kb + G.Bd - 1) / G.Bd);

  for (int b = tid; b < kHistBins; b += T) hist[b] = 0u;  // used after later barriers
  if (tid == 0) {
    sh.mm[0] = sh.mm[1] = 0u;
    sh.arrived = 0u;
  }
  uint32_t ab[kElemsPerThread];
  dequant_block(gv, cv, sh.levels, ab);
  if (L < kElemsPerThread * T) {  // slots past the block's end hold +0
#pragma unroll
    for (int c = 0; c < kChunks; ++c)
#pragma unroll
      for (int e = 0; e < kChunk; ++e)
        if (elem_index<T>(c, tid, e) >= L) ab[c * kChunk + e] = 0u;
  }

  uint32_t* row = A.window + ((int64_t)j * G.m + A.row) * G.kp;
  float rmin = 0.0f, rmax = 0.0f;  // selected entries become +0
  bool listed = false;

  // (2) candidate tier. tau_lo: a high order statistic of the warps' top-2
  // samples (one sample per thread, stride 8); every warp sorts the 2*NW
  // values itself, so no broadcast barrier is needed.
  const int r_target = (5 * k + 63) / 64;
  if (8 * k <= L && r_target <= min(2 * NW, 32)) {
    const uint32_t s = ab[0] & 0x7FFFFFFFu;
    uint32_t m1 = s;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m1 = max(m1, __shfl_xor_sync(0xFFFFFFFFu, m1, o));
    const int first = __ffs(__ballot_sync(0xFFFFFFFFu, s == m1)) - 1;
    uint32_t m2 = (lane == first) ? 0u : s;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m2 = max(m2, __shfl_xor_sync(0xFFFFFFFFu, m2, o));
    if (lane == 0) {
      sh.top[2 * wid] = m1;
      sh.top[2 * wid + 1] = m2;
    }
    __syncthreads();
    uint32_t v = (lane < 2 * NW) ? sh.top[lane] : 0u;
#pragma unroll
    for (int size = 2; size <= 32; size <<= 1) {  // bitonic sort, descending
#pragma unroll
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        const uint32_t o = __shfl_xor_sync(0xFFFFFFFFu, v, stride);
        const bool up = ((lane & size) == 0);
        const bool lower = ((lane & stride) == 0);
        v = (lower == up) ? max(v, o) : min(v, o);
      }
    }
    const uint32_t tau_lo = __shfl_sync(0xFFFFFFFFu, v, r_target - 1);

    // Counts of candidates per chunk (16-bit fields), residual min/max of the
    // rest, and the largest key.
    unsigned long long pc = 0ull;
    uint32_t kmax = 0u;
#pragma unroll
    for (int c = 0; c < kChunks; ++c) {
      uint32_t cnt = 0;
#pragma unroll
      for (int e = 0; e < kChunk; ++e) {
        const uint32_t bits = ab[c * kChunk + e];
        const uint32_t key = bits & 0x7FFFFFFFu;
        const bool cand = key >= tau_lo;
        cnt += cand;
        kmax = max(kmax, key);
        const float v = cand ? 0.0f : __uint_as_float(bits);
        rmin = fminf(rmin, v);
        rmax = fmaxf(rmax, v);
      }
      pc |= (unsigned long long)cnt << (16 * c);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) kmax = max(kmax, __shfl_xor_sync(0xFFFFFFFFu, kmax, o));
    if (lane == 0) sh.wmax[wid] = kmax;
    unsigned long long tot;
    const unsigned long long x = block_scan_1bar<T, unsigned long long>(pc, sh.scan64, tot) - pc;
    kmax = (lane < NW) ? sh.wmax[lane] : 0u;  // written before the scan's barrier
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) kmax = max(kmax, __shfl_xor_sync(0xFFFFFFFFu, kmax, o));
    if (tid == 0 && kmax >= 0x7F800000u) atomicOr(&A.hdr[kHdrStatus], kStatusNonFinite);
    int n = 0;
#pragma unroll
    for (int c = 0; c < kChunks; ++c) n += (int)((tot >> (16 * c)) & 0xFFFFu);

    if (n >= k && n <= kCandCap) {
      uint32_t base = 0;
#pragma unroll
      for (int c = 0; c < kChunks; ++c) {
        uint32_t run = base + (uint32_t)((x >> (16 * c)) & 0xFFFFu);
        base += (uint32_t)((tot >> (16 * c)) & 0xFFFFu);
#pragma unroll
        for (int e = 0; e < kChunk; ++e) {
          const uint32_t bits = ab[c * kChunk + e];
          const bool cand = (bits & 0x7FFFFFFFu) >= tau_lo;
          if (cand) {  // n <= kCandCap bounds run
            cab[run] = bits;
            cidx[run] = (uint16_t)elem_index<T>(c, tid, e);
          }
          run += cand;
        }
      }
      __syncthreads();
      select_list<T>(cab, cidx, n, k, tau_lo, kmax, hist, sh, row, rmin, rmax);
      listed = true;
    } else {
      rmin = rmax = 0.0f;
    }
  }
  if (!listed) {
    // (2) full tier.
    select_full<T, VEC>(A.grads, A.codes, A.hdr, start, L, k, sh.levels, hist, sh, row, rmin,
                        rmax);
  }
  for (int sl = k + tid; sl < G.kp; sl += T) row[sl] = kEmptySlot;
  block_minmax_to_global<T>(rmin, rmax, sh, A.hdr, A.pair_next);

  // (6) for this kernel's share of the blocks; the row above is complete.
  if (update_in_select(A, j)) {
    __syncthreads();
    block_update<T>(A, j, start, L, work, sh.w1, sh.w2);
  }
}

// One CTA per block.
template <int T, bool VEC>
__global__ void __launch_bounds__(T, (T <= 512 ? 1024 / T : 1))
    mua_select_kernel(const __grid_constant__ StepArgs A) {
  extern __shared__ __align__(128) uint8_t dyn[];
  __shared__ SelectShared sh;
  const int j = blockIdx.x;
  int64_t start;
  int L;
  block_span(A, j, start, L);
  uint4 gv[kChunks];
  uint32_t cv[kChunks];
  load_block<T, VEC>(A.grads, A.codes, start, L, threadIdx.x, gv, cv);
  {  // (1) the 16 levels of Q^{-1}(e_t, delta_t, Delta_t)
    const float delta = 0.0f - __uint_as_float(A.hdr[A.pair_cur]);
    const float Delta = __uint_as_float(A.hdr[A.pair_cur + 1]);
    fill_levels(sh.levels, delta, __fdiv_rn(__fsub_rn(Delta, delta), 15.0f));
  }
  load_weights(A, sh.w1, sh.w2);
  __syncthreads();
  select_block<T, VEC>(A, j, gv, cv, dyn, sh);
}

// Persistent CTAs (B_d % 32 == 0): each CTA walks the blocks
// j = blockIdx.x + i * gridDim.x. One shared-memory stage holds a block's
// gradients and codes, filled by bulk copies (TMA): as soon as the threads
// have moved block i into registers, the copy of block i+1 is issued, so it
// lands while block i is processed. A ragged last block is read directly.
// Shared memory: stage {bf16 g[B_d], codes[B_d/2]}, then `work`.
template <int T>
__global__ void __launch_bounds__(T, (T <= 512 ? 1024 / T : 1))
    mua_select_persistent(const __grid_constant__ StepArgs A) {
  extern __shared__ __align__(128) uint8_t dyn[];
  __shared__ SelectShared sh;
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint32_t s_fail;
  const Geometry& G = A.g;
  const int tid = threadIdx.x;
  const uint32_t gbytes = 2u * (uint32_t)G.Bd, cbytes = (uint32_t)G.Bd / 2u;
  const uint32_t stage_bytes = (gbytes + cbytes + 127u) & ~127u;
  uint8_t* work = dyn + stage_bytes;
  const int nfull = (G.last_len == G.Bd) ? G.nb : G.nb - 1;  // blocks fed by TMA
  const int step = gridDim.x;

  auto issue = [&](int jj) {  // one thread: stage <- block jj
    fence_proxy_async();
    mbar_expect_tx(&bar, gbytes + cbytes);
    bulk_g2s(dyn, A.grads + (int64_t)jj * G.Bd, gbytes, &bar);
    bulk_g2s(dyn + gbytes, A.codes + ((int64_t)jj * G.Bd >> 1), cbytes, &bar);
  };
  if (tid == 0) {
    mbar_init(&bar, 1);
    mbar_init_fence();
    s_fail = 0u;
  }
  {  // (1) the 16 levels of Q^{-1}(e_t, delta_t, Delta_t)
    const float delta = 0.0f - __uint_as_float(A.hdr[A.pair_cur]);
    const float Delta = __uint_as_float(A.hdr[A.pair_cur + 1]);
    fill_levels(sh.levels, delta, __fdiv_rn(__fsub_rn(Delta, delta), 15.0f));
  }
  load_weights(A, sh.w1, sh.w2);
  __syncthreads();
  if (tid == 0 && (int)blockIdx.x < nfull) issue(blockIdx.x);
  uint32_t uses = 0;      // completed phases of `bar`
  bool in_flight = (int)blockIdx.x < nfull;
  for (int i = 0;; ++i) {
    const int j = blockIdx.x + i * step;
    if (j >= G.nb) break;
    uint4 gv[kChunks];
    uint32_t cv[kChunks];
    if (j < nfull) {
      if (!mbar_wait(&bar, uses & 1u)) atomicOr(&s_fail, 1u);
      __syncthreads();
      if (s_fail) break;
      ++uses;
      in_flight = false;
      load_block_smem<T>(reinterpret_cast<const uint16_t*>(dyn), dyn + gbytes, tid, gv, cv);
      __syncthreads();  // every thread has read the stage: refill it
      const int jn = j + step;
      if (jn < nfull) {
        if (tid == 0) issue(jn);
        in_flight = true;
      }
    } else {
      load_block<T, true>(A.grads, A.codes, (int64_t)j * G.Bd, G.last_len, tid, gv, cv);
    }
    select_block<T, true>(A, j, gv, cv, work, sh);
    __syncthreads();  // `work` is reused by the next block
  }
  if (s_fail) {
    // A wait gave up: record it and give the copy still in flight a bounded
    // chance to land before the CTA's shared memory is released.
    if (tid == 0) {
      atomicOr(&A.hdr[kHdrStatus], kStatusTimeout);
      if (in_flight) (void)mbar_wait(&bar, uses & 1u);
    }
    __syncthreads();
  }
}

template <int T>
cudaError_t launch_t(const StepArgs& args, bool vec, bool persistent, uint32_t smem,
                     cudaStream_t stream) {
  if (persistent) {
    auto kern = mua_select_persistent<T>;
    // must match the kernel: bf16 g[B_d] + codes[B_d/2], rounded up to 128 bytes
    const uint32_t stage = (2u * (uint32_t)args.g.Bd + (uint32_t)args.g.Bd / 2u + 127u) & ~127u;
    const uint32_t total = stage + smem;
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)total);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0, per_sm = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return e;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, T, total)) !=
        cudaSuccess)
      return e;
    const int grid = (int)std::min<int64_t>(args.g.nb, (int64_t)std::max(1, per_sm) * sms);
    kern<<<grid, T, total, stream>>>(args);
    return cudaGetLastError();
  }
  auto kern = vec ? mua_select_kernel<T, true> : mua_select_kernel<T, false>;
  if (smem > 32 * 1024) {  // opt in well below 48 KB: static arrays count too
    const cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  kern<<<args.g.nb, T, smem, stream>>>(args);
  return cudaGetLastError();
}

}  // namespace

uint32_t select_smem_bytes(int threads, int Bd, int kp, int m) {
  const uint32_t own = 4u * kHistBins + 6u * kCandCap;
  const uint32_t upd = update_smem_bytes(threads, Bd, kp, m);
  return own > upd ? own : upd;
}

cudaError_t launch_select(const StepArgs& args, int threads, bool vec, bool persistent,
                          uint32_t smem, cudaStream_t stream) {
  switch (threads) {
    case 32: return launch_t<32>(args, vec, persistent, smem, stream);
    case 64: return launch_t<64>(args, vec, persistent, smem, stream);
    case 128: return launch_t<128>(args, vec, persistent, smem, stream);
    case 256: return launch_t<256>(args, vec, persistent, smem, stream);
    case 512: return launch_t<512>(args, vec, persistent, smem, stream);
    case 1024: return launch_t<1024>(args, vec, persistent, smem, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace mua
