// Stage kernel 1 of the MicroAdam step, one WARP per block ([MicroAdam ¶1] =
// paragraph 1 of "MicroAdam (Sparse-Gradient Adaptive Optimization with
// Quantized Error Feedback)"):
//   a_t = g_t + Q^{-1}(e_t, delta_t, Delta_t)      (streamed, never stored)
//   (I_t, V_t) = Top-k of |a_t| (ties to the lower index), written in
//   ascending index order to row t mod m of the window G,
//   the residual's block min/max folded into the global (-delta_{t+1},
//   Delta_{t+1}) pair with one pair of integer atomics per block.
//
// The blocks are independent, so a warp (not a CTA) owns one: no block-wide
// barrier, few registers and a few KB of shared memory per warp, so tens of
// blocks are in flight per SM and memory latency hides behind the others.
//
// Exact Top-k:
//  * candidate path (blocks of 1024 to 32768 entries): 512 sample keys (64
//    chunks of 8 spread over the block), each lane's top-2, a warp sort of
//    those 64 values -> tau_lo (aiming at ~2.5k candidates over the block);
//    one streaming pass (lane l holds elements 256 s + 8 l .. + 7 of step s)
//    appends every
//    |a| >= tau_lo to the lane's own strided region of the list, with no
//    cross-lane step, and folds the rest into the residual min/max; an exact
//    warp radix select on the list (8-bit digits from the highest bit where
//    tau_lo and the list maximum differ) finds the k-th key; the selected
//    entries are marked in a bitmask of the block (ties at the threshold by a
//    lowest-index merge of the lanes' regions, each already in index order)
//    and a popcount prefix of the mask gives each its place in the row;
//  * fallback (blocks under 1024 entries, k > L/8, too few candidates after
//    the retry, or a lane that dropped a key at or above the threshold):
//    exact radix select on all keys by streaming passes over the block (it
//    is in L2 by then), 8 bits per pass, then one placing pass.
// HBM traffic per parameter: 2 B gradient + 0.5 B codes read; per selected
// entry 4 B written.
#include "mua_kernels.cuh"

namespace mua {
namespace {

constexpr int kWarps = 8;         // warps (= blocks in flight) per CTA
constexpr int kWarpCap = 1024;    // candidate list entries per warp
constexpr int kLaneCap = kWarpCap / 32;  // entries per lane region
constexpr int kUnroll = 4;        // 256-element steps loaded ahead

// MASKW: words of the selection bitmask, which covers one block (512 for
// blocks of up to 16384 entries, 1024 up to 32768).
template <int MASKW>
struct WarpSmem {
  uint32_t bits[kWarpCap];  // a_t bits; lane l's i-th candidate at [32 i + l]
  uint16_t idx[kWarpCap];   // its block-relative index
  uint32_t hist[MASKW / 2 > 256 ? MASKW / 2 : 256];  // radix histogram, then the
                                                     // mask's u16 word prefix
  uint32_t mask[MASKW];
};

template <int MASKW>
struct CtaSmem {
  float levels[16];
  WarpSmem<MASKW> w[kWarps];
};

__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t x, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  return x;
}

// One 256-element step: lane l holds elements base + 8 l .. + 7 of the block
// (bits of a_t; +0 past L).
template <bool VEC>
__device__ __forceinline__ void load_step(const uint16_t* __restrict__ grads,
                                          const uint8_t* __restrict__ codes, int64_t start,
                                          int L, int e0, uint4& gv, uint32_t& cv) {
  if (VEC && e0 + kChunk <= L) {
    gv = ld_stream_v4(grads + start + e0);
    cv = ld_stream_u32(codes + ((start + e0) >> 1));
  } else {
    uint32_t w[4] = {0u, 0u, 0u, 0u};
    uint32_t cw = 0u;
#pragma unroll
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
}

__device__ __forceinline__ void dequant8(const uint4& gv, uint32_t cv, const float* lv, int e0,
                                         int L, uint32_t (&ab)[kChunk]) {
#pragma unroll
  for (int e = 0; e < kChunk; ++e) {
    const float a = __fadd_rn(__uint_as_float(grad_bits(gv, e)), lv[(cv >> (4 * e)) & 0xFu]);
    ab[e] = (e0 + e < L) ? __float_as_uint(a) : 0u;
  }
}

// dequant8 for a step wholly inside the block. The code word is pre-scaled by 4
// so each nibble becomes a byte offset into the level table directly.
__device__ __forceinline__ void dequant8_full(const uint4& gv, uint32_t cv, const float* lv,
                                              uint32_t (&ab)[kChunk]) {
  const uint32_t c4 = cv << 2;
  const char* lb = reinterpret_cast<const char*>(lv);
#pragma unroll
  for (int e = 0; e < kChunk; ++e) {
    const uint32_t off = (e == 0) ? (c4 & 0x3Cu) : ((cv >> (4 * e - 2)) & 0x3Cu);
    const float a = __fadd_rn(__uint_as_float(grad_bits(gv, e)),
                              *reinterpret_cast<const float*>(lb + off));
    ab[e] = __float_as_uint(a);
  }
}

// Per-lane state of the candidate pass.
struct LaneState {
  uint32_t cnt;  // entries in the lane's region
  uint32_t tau;  // candidate threshold of the lane (>= the warp's tau_lo)
  float rmin, rmax;
};

// Makes room in a lane's region for one more 8-element step: while it holds
// more than kLaneCap - 8 entries, the smallest is dropped into the residual's
// min/max (its slot takes the region's last entry) and the lane's threshold
// rises above it, so every key the lane ever drops is below its final tau.
__device__ __forceinline__ LaneState make_room(uint32_t* bits, uint16_t* idx, int lane,
                                            LaneState st) {
  while (st.cnt > (uint32_t)(kLaneCap - kChunk)) {
    uint32_t m0 = 0xFFFFFFFFu, at = 0u;
    for (uint32_t i = 0; i < st.cnt; ++i) {
      const uint32_t key = bits[32 * i + lane] & 0x7FFFFFFFu;
      if (key < m0) {
        m0 = key;
        at = i;
      }
    }
    const float v = __uint_as_float(bits[32 * at + lane]);
    st.rmin = fminf(st.rmin, v);
    st.rmax = fmaxf(st.rmax, v);
    st.tau = max(st.tau, m0 + 1u);
    const uint32_t last = st.cnt - 1u;
    bits[32 * at + lane] = bits[32 * last + lane];
    idx[32 * at + lane] = idx[32 * last + lane];
    st.cnt = last;
  }
  return st;
}

__device__ __forceinline__ void put_row(uint32_t* row, uint32_t pos, int k, uint32_t idx,
                                        uint32_t abits) {
  if (pos < (uint32_t)k) {
    const uint32_t vb = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(abits)));
    row[pos] = (idx & 0xFFFFu) | (vb << 16);
  }
}

// Finds, in a warp-private histogram of nbins (<= 256) counts, the bin holding
// the krem-th largest key. Lane l owns bins [8 l, 8 l + 8).
__device__ __forceinline__ void warp_find_bin(const uint32_t* hist, int nbins, int krem,
                                              int lane, uint32_t& bin, uint32_t& above,
                                              uint32_t& inbin) {
  const int b0 = lane * 8;
  uint32_t h[8];
  uint32_t own = 0;
#pragma unroll
  for (int b = 0; b < 8; ++b) {
    h[b] = (b0 + b < nbins) ? hist[b0 + b] : 0u;
    own += h[b];
  }
  const uint32_t incl = warp_incl_scan(own, lane);
  uint32_t running = __shfl_sync(0xFFFFFFFFu, incl, 31) - incl;  // bins above this lane
  bool found = false;
  uint32_t fb = 0u, fa = 0u, fi = 0u;
#pragma unroll
  for (int b = 7; b >= 0; --b) {
    if (!found && running < (uint32_t)krem && running + h[b] >= (uint32_t)krem) {
      found = true;
      fb = (uint32_t)(b0 + b);
      fa = running;
      fi = h[b];
    }
    running += h[b];
  }
  const int src = __ffs(__ballot_sync(0xFFFFFFFFu, found)) - 1;
  bin = __shfl_sync(0xFFFFFFFFu, fb, src & 31);
  above = __shfl_sync(0xFFFFFFFFu, fa, src & 31);
  inbin = __shfl_sync(0xFFFFFFFFu, fi, src & 31);
}

// Exact selection threshold among keys that all share the bits of `prefix`
// above bit hi (keys come from `key_of(i)`, i in the lane's entries). On
// return: mode 0 -> selected = key >= thr; mode 1 -> key > thr, or key == thr
// for the `need` lowest indices.
template <typename KeyAt>
__device__ __forceinline__ void warp_radix(int hi, uint32_t prefix, int k, uint32_t* hist,
                                           int lane, KeyAt&& for_each_key, int& mode,
                                           uint32_t& thr, int& need) {
  uint32_t pmask = (hi >= 30) ? 0u : ((0xFFFFFFFFu << (hi + 1)) & 0x7FFFFFFFu);
  prefix &= pmask;
  int krem = k;
  mode = 1;
  while (hi >= 0) {
    const int width = min(8, hi + 1);
    const int shift = hi + 1 - width;
    const int nbins = 1 << width;
#pragma unroll
    for (int b = 0; b < 8; ++b) hist[lane * 8 + b] = 0u;
    __syncwarp();
    for_each_key([&](uint32_t key) {
      if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & (nbins - 1)], 1u);
    });
    __syncwarp();
    uint32_t bin, above, inbin;
    warp_find_bin(hist, nbins, krem, lane, bin, above, inbin);
    __syncwarp();
    prefix |= bin << shift;
    pmask |= (uint32_t)(nbins - 1) << shift;
    krem -= (int)above;
    hi = shift - 1;
    if (inbin == (uint32_t)krem) {  // the whole bin is selected
      mode = 0;
      thr = prefix;
      need = k;
      return;
    }
  }
  thr = prefix;
  need = krem;
}

template <bool VEC, int MASKW>
__global__ void __launch_bounds__(kWarps * 32, 3)
    mua_select_warp_kernel(const __grid_constant__ StepArgs A) {
  extern __shared__ __align__(16) uint8_t dyn[];
  CtaSmem<MASKW>& S = *reinterpret_cast<CtaSmem<MASKW>*>(dyn);
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const Geometry& G = A.g;
  {
    const float delta = 0.0f - __uint_as_float(A.hdr[A.pair_cur]);
    const float Delta = __uint_as_float(A.hdr[A.pair_cur + 1]);
    fill_levels(S.levels, delta, __fdiv_rn(__fsub_rn(Delta, delta), 15.0f));
  }
  __syncthreads();  // the only CTA barrier: the level table
  const int j = blockIdx.x * kWarps + wid;
  if (j >= G.nb) return;
  WarpSmem<MASKW>& W = S.w[wid];
  const float* lv = S.levels;
  int64_t start;
  int L;
  block_span(A, j, start, L);
  const int k = (int)(((int64_t)L * G.kb + G.Bd - 1) / G.Bd);
  uint32_t* row = A.window + ((int64_t)j * G.m + A.row) * G.kp;
  const int nsteps = (L + 255) >> 8;

  float rmin = 0.0f, rmax = 0.0f;  // residual; selected entries become +0
  bool done = false;

  // ---------------- candidate path
  if (L >= 1024 && L <= 32 * MASKW && 8 * k <= L) {
    // 512 samples: 64 chunks of 8, chunk c at element (c * (L / 64)) & ~7.
    const int cstride = (L / 64) & ~7;
    uint32_t t1 = 0u, t2 = 0u;  // this lane's two largest sample keys
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int e0 = (lane + 32 * h) * cstride;
      uint4 gv;
      uint32_t cv;
      load_step<VEC>(A.grads, A.codes, start, L, e0, gv, cv);
      uint32_t ab[kChunk];
      dequant8(gv, cv, lv, e0, L, ab);
#pragma unroll
      for (int e = 0; e < kChunk; ++e) {
        const uint32_t key = ab[e] & 0x7FFFFFFFu;
        const uint32_t lo = min(t1, key);
        t1 = max(t1, key);
        t2 = max(t2, lo);
      }
    }
    // bitonic sort of the 64 values (2 per lane), descending; element r of the
    // sorted order lives in lane r / 2, slot r % 2.
    uint32_t v0 = max(t1, t2), v1 = min(t1, t2);
#pragma unroll
    for (int size = 2; size <= 64; size <<= 1) {
#pragma unroll
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        if (stride == 1) {  // within the lane: elements 2 lane, 2 lane + 1
          const bool up = (((2 * lane) & size) == 0);
          const uint32_t hi2 = max(v0, v1), lo2 = min(v0, v1);
          v0 = up ? hi2 : lo2;
          v1 = up ? lo2 : hi2;
        } else {
          const int ls = stride >> 1;  // lane distance
          const uint32_t o0 = __shfl_xor_sync(0xFFFFFFFFu, v0, ls);
          const uint32_t o1 = __shfl_xor_sync(0xFFFFFFFFu, v1, ls);
          const bool up = (((2 * lane) & size) == 0);
          const bool lower = ((lane & ls) == 0);
          const bool keep_max = (lower == up);
          v0 = keep_max ? max(v0, o0) : min(v0, o0);
          v1 = keep_max ? max(v1, o1) : min(v1, o1);
        }
      }
    }
    // rank of tau_lo among the 64: ~2.5k candidates expected over the block
    const int r = min(63, (int)((1280 * (int64_t)k + L - 1) / L) - 1);
    const uint32_t tl0 = __shfl_sync(0xFFFFFFFFu, v0, r >> 1);
    const uint32_t tl1 = __shfl_sync(0xFFFFFFFFu, v1, r >> 1);
    const uint32_t tau_first = (r & 1) ? tl1 : tl0;
    const uint32_t tau_retry = __shfl_sync(0xFFFFFFFFu, v1, 31);  // smallest of the 64

    // One streaming pass per attempt (a second, with a lower tau_lo, only when
    // the first finds fewer than k candidates).
    for (int attempt = 0; attempt < 2 && !done; ++attempt) {
      const uint32_t tau_lo = attempt == 0 ? tau_first : tau_retry;
      if (attempt == 1 && tau_retry >= tau_first) break;
      // Candidates (key >= tau) go to the lane's region. Before each step a
      // lane with fewer than 8 free slots drops its smallest entries and
      // raises its tau (make_room), so a step's appends always fit. The
      // result is exact when every raised tau is at most the final
      // threshold (checked below).
      LaneState ls{0u, tau_lo, 0.0f, 0.0f};
      auto scan_step = [&](const uint32_t (&ab)[kChunk], int e0, bool full) {
        if (__any_sync(0xFFFFFFFFu, ls.cnt > (uint32_t)(kLaneCap - kChunk))) {
          if (ls.cnt > (uint32_t)(kLaneCap - kChunk)) ls = make_room(W.bits, W.idx, lane, ls);
          __syncwarp();
        }
#pragma unroll
        for (int e = 0; e < kChunk; ++e) {
          const uint32_t key = ab[e] & 0x7FFFFFFFu;
          const bool cand = key >= ls.tau && (full || e0 + e < L);
          if (cand) {
            W.bits[(ls.cnt << 5) | (uint32_t)lane] = ab[e];
            W.idx[(ls.cnt << 5) | (uint32_t)lane] = (uint16_t)(e0 + e);
          }
          ls.cnt += cand ? 1u : 0u;
          const float v = cand ? 0.0f : __uint_as_float(ab[e]);
          ls.rmin = fminf(ls.rmin, v);
          ls.rmax = fmaxf(ls.rmax, v);
        }
      };
      const int nfull = L >> 8;  // steps with all 256 elements inside the block
      for (int s0 = 0; s0 < nfull; s0 += kUnroll) {
        uint4 gv[kUnroll];
        uint32_t cv[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          const int e0 = ((s0 + u) << 8) + 8 * lane;
          if (s0 + u < nfull) load_step<VEC>(A.grads, A.codes, start, L, e0, gv[u], cv[u]);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          if (s0 + u >= nfull) break;
          uint32_t ab[kChunk];
          dequant8_full(gv[u], cv[u], lv, ab);
          scan_step(ab, ((s0 + u) << 8) + 8 * lane, true);
        }
      }
      if (nfull < nsteps) {  // the block's partial last step
        const int e0 = (nfull << 8) + 8 * lane;
        uint4 gv;
        uint32_t cv;
        load_step<VEC>(A.grads, A.codes, start, L, e0, gv, cv);
        uint32_t ab[kChunk];
        dequant8(gv, cv, lv, e0, L, ab);
        scan_step(ab, e0, false);
      }
      rmin = ls.rmin;
      rmax = ls.rmax;
      const uint32_t cnt = ls.cnt;
      const int mine = (int)cnt;
      const uint32_t n = __reduce_add_sync(0xFFFFFFFFu, cnt);
      const uint32_t drop_bound = __reduce_max_sync(0xFFFFFFFFu, ls.tau > tau_lo ? ls.tau : 0u);
      __syncwarp();
      if (n < (uint32_t)k) continue;  // too few: retry lower, else the fallback
      uint32_t kmax = 0u;
      for (int i = 0; i < mine; ++i) kmax = max(kmax, W.bits[32 * i + lane] & 0x7FFFFFFFu);
      kmax = __reduce_max_sync(0xFFFFFFFFu, kmax);
      int mode = 1, need = k;
      uint32_t thr = tau_lo;
      const uint32_t diff = kmax ^ tau_lo;
      if (diff != 0u) {
        warp_radix(31 - __clz(diff), tau_lo, k, W.hist, lane,
                   [&](auto&& f) {
                     for (int i = 0; i < mine; ++i) f(W.bits[32 * i + lane] & 0x7FFFFFFFu);
                   },
                   mode, thr, need);
      }
      // Exact only if every dropped key (< its lane's tau <= drop_bound) is below thr.
      if (drop_bound > thr) break;
      if (lane == 0 && kmax >= 0x7F800000u) atomicOr(&A.hdr[kHdrStatus], kStatusNonFinite);
      // Selection bitmask: keys above the threshold (at or above it in mode 0) ...
      const int wn = (L + 31) >> 5;
      for (int w = lane; w < wn; w += 32) W.mask[w] = 0u;
      __syncwarp();
      for (int i = 0; i < mine; ++i) {
        const uint32_t key = W.bits[32 * i + lane] & 0x7FFFFFFFu;
        if (mode == 0 ? key >= thr : key > thr) {
          const uint32_t idx = W.idx[32 * i + lane];
          atomicOr(&W.mask[idx >> 5], 1u << (idx & 31));
        }
      }
      // ... and, in mode 1, the `need` lowest indices among keys equal to it,
      // one per round: the lowest unmarked tied index over all lanes.
      if (mode == 1) {
        for (int q = 0; q < need; ++q) {
          __syncwarp();
          uint32_t head = 0xFFFFu;
          for (int i = 0; i < mine; ++i) {
            if ((W.bits[32 * i + lane] & 0x7FFFFFFFu) != thr) continue;
            const uint32_t idx = W.idx[32 * i + lane];
            if (idx < head && !((W.mask[idx >> 5] >> (idx & 31)) & 1u)) head = idx;
          }
          const uint32_t low = __reduce_min_sync(0xFFFFFFFFu, head);
          if (head == low && head != 0xFFFFu) atomicOr(&W.mask[head >> 5], 1u << (head & 31));
        }
      }
      __syncwarp();
      // u16 exclusive popcount prefix of the mask words (lane l: words
      // MASKW/32 l ..)
      uint16_t* wpre = reinterpret_cast<uint16_t*>(W.hist);
      {
        constexpr int kWpl = MASKW / 32;
        const int w0 = kWpl * lane;
        uint32_t c = 0u;
#pragma unroll
        for (int w = 0; w < kWpl; ++w) c += (w0 + w < wn) ? (uint32_t)__popc(W.mask[w0 + w]) : 0u;
        uint32_t run = warp_incl_scan(c, lane) - c;
#pragma unroll
        for (int w = 0; w < kWpl; ++w) {
          if (w0 + w < wn) {
            wpre[w0 + w] = (uint16_t)run;
            run += (uint32_t)__popc(W.mask[w0 + w]);
          }
        }
      }
      __syncwarp();
      // Place the selected entries; the others join the residual's min/max.
      for (int i = 0; i < mine; ++i) {
        const uint32_t bits = W.bits[32 * i + lane];
        const uint32_t idx = W.idx[32 * i + lane];
        const uint32_t word = W.mask[idx >> 5];
        if ((word >> (idx & 31)) & 1u) {
          const uint32_t pos = wpre[idx >> 5] + (uint32_t)__popc(word & ((1u << (idx & 31)) - 1u));
          put_row(row, pos, k, idx, bits);
        } else {
          rmin = fminf(rmin, __uint_as_float(bits));
          rmax = fmaxf(rmax, __uint_as_float(bits));
        }
      }
      done = true;
    }
  }

  // ---------------- fallback: streaming radix select over the whole block
  if (!done) {
    rmin = rmax = 0.0f;
    int mode, need;
    uint32_t thr;
    auto stream_keys = [&](auto&& f) {
      for (int s = 0; s < nsteps; ++s) {
        const int e0 = (s << 8) + 8 * lane;
        uint4 gv;
        uint32_t cv;
        load_step<VEC>(A.grads, A.codes, start, L, e0, gv, cv);
        uint32_t ab[kChunk];
        dequant8(gv, cv, lv, e0, L, ab);
#pragma unroll
        for (int e = 0; e < kChunk; ++e) f(ab[e] & 0x7FFFFFFFu);
      }
    };
    warp_radix(30, 0u, k, W.hist, lane, stream_keys, mode, thr, need);
    uint32_t run_g = 0u, run_e = 0u;  // warp-uniform running counts
    uint32_t kmax = 0u;
    for (int s = 0; s < nsteps; ++s) {
      const int e0 = (s << 8) + 8 * lane;
      uint4 gv;
      uint32_t cv;
      load_step<VEC>(A.grads, A.codes, start, L, e0, gv, cv);
      uint32_t ab[kChunk];
      dequant8(gv, cv, lv, e0, L, ab);
      uint32_t cg = 0u, ce = 0u;
#pragma unroll
      for (int e = 0; e < kChunk; ++e) {
        const uint32_t key = ab[e] & 0x7FFFFFFFu;
        if (e0 + e >= L) continue;
        kmax = max(kmax, key);
        if (mode == 0) {
          cg += key >= thr;
        } else {
          cg += key > thr;
          ce += key == thr;
        }
      }
      const uint32_t packed = cg | (ce << 16);
      const uint32_t incl = warp_incl_scan(packed, lane);
      const uint32_t tot = __shfl_sync(0xFFFFFFFFu, incl, 31);
      uint32_t g = run_g + ((incl - packed) & 0xFFFFu);
      uint32_t q = run_e + ((incl - packed) >> 16);
#pragma unroll
      for (int e = 0; e < kChunk; ++e) {
        const uint32_t bits = ab[e];
        const uint32_t key = bits & 0x7FFFFFFFu;
        const bool gt = (mode == 0) ? key >= thr : key > thr;
        if (e0 + e >= L) continue;
        if (gt) {
          put_row(row, g + min(q, (uint32_t)need), k, (uint32_t)(e0 + e), bits);
          ++g;
        } else if (mode == 1 && key == thr && q < (uint32_t)need) {
          put_row(row, g + q, k, (uint32_t)(e0 + e), bits);
          ++q;
        } else {
          if (mode == 1 && key == thr) ++q;
          rmin = fminf(rmin, __uint_as_float(bits));
          rmax = fmaxf(rmax, __uint_as_float(bits));
        }
      }
      run_g += tot & 0xFFFFu;
      run_e += tot >> 16;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) kmax = max(kmax, __shfl_xor_sync(0xFFFFFFFFu, kmax, o));
    if (lane == 0 && kmax >= 0x7F800000u) atomicOr(&A.hdr[kHdrStatus], kStatusNonFinite);
  }

  for (int sl = k + lane; sl < G.kp; sl += 32) row[sl] = kEmptySlot;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    rmin = fminf(rmin, __shfl_xor_sync(0xFFFFFFFFu, rmin, o));
    rmax = fmaxf(rmax, __shfl_xor_sync(0xFFFFFFFFu, rmax, o));
  }
  if (lane == 0) {
    atomicMax(&A.hdr[A.pair_next], __float_as_uint(0.0f - rmin));  // >= +0, canonical zero
    atomicMax(&A.hdr[A.pair_next + 1], __float_as_uint(rmax + 0.0f));
  }
}

}  // namespace

uint32_t select_warp_smem_bytes(int Bd) {
  return Bd <= 16384 ? (uint32_t)sizeof(CtaSmem<512>) : (uint32_t)sizeof(CtaSmem<1024>);
}

cudaError_t launch_select_warp(const StepArgs& args, bool vec, cudaStream_t stream) {
  const bool big = args.g.Bd > 16384;
  auto kern = big ? (vec ? mua_select_warp_kernel<true, 1024> : mua_select_warp_kernel<false, 1024>)
                  : (vec ? mua_select_warp_kernel<true, 512> : mua_select_warp_kernel<false, 512>);
  const uint32_t smem = select_warp_smem_bytes(args.g.Bd);
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = (args.g.nb + kWarps - 1) / kWarps;
  kern<<<grid, kWarps * 32, smem, stream>>>(args);
  return cudaGetLastError();
}

}  // namespace mua
