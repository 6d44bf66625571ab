// Stage kernel 1 of the MicroAdam step, one WARP per block ([MicroAdam ¶1] =
// paragraph 1 of "MicroAdam (Sparse-Gradient Adaptive Optimization with
// Quantized Error Feedback)"):
//   a_t = g_t + Q^{-1}(e_t, delta_t, Delta_t)      (streamed, never stored)
//   (I_t, V_t) = Top-k of |a_t| (ties to the lower index), written to row
//   t mod m of the window G,
//   the residual's block min/max folded into the global (-delta_{t+1},
//   Delta_{t+1}) pair with one pair of integer atomics per block.
// The order of the k pairs inside a row is not part of the method (the
// AdamStats sums run per index, row by row); the kernel's order is fixed by
// the data alone (see the candidate path).
//
// The blocks are independent, so a warp (not a CTA) owns one: no block-wide
// barrier, and memory latency hides behind the other warps' blocks. A CTA is
// one warp by default: its shared memory is released as soon as its block is
// done, whatever the other blocks on the SM take.
//
// Exact Top-k:
//  * candidate path (blocks of 1024 to LMAX entries, k <= L/8):
//    512 sample keys (64 chunks of 8 spread over the block), each lane's top
//    two, a warp sort of those 64 values -> tau_lo. One streaming pass (lane l
//    holds elements 256 s + 8 l .. + 7 of step s) tests each |a| against the
//    lane's threshold and appends the candidates {bits of a, index} to the
//    lane's own strided region with one predicated 4-byte and one 2-byte
//    store; nothing else happens per element. A lane whose region fills
//    drops its smallest keys and raises its threshold above them
//    (make_room). An exact warp radix select over the candidates (8-bit
//    digits from the highest bit where tau_lo and the largest candidate
//    differ) gives the k-th key; the result is exact iff every raised lane
//    threshold is at most that key (else the block takes the fallback). Ties
//    at the threshold go to the lowest indices by a merge of the lanes'
//    regions (each ascends by index). The row holds lane 0's selected entries,
//    then lane 1's, ..., each lane's in ascending index order;
//  * residual min/max without a per-element cost: an element a lane did not
//    append has |a| below that lane's final threshold. The candidates that
//    were not selected (and the dropped ones) are folded into the block's min
//    and max; if those reach past +-tau_lo, only the elements of lanes that
//    raised their threshold beyond them can still change the result, and the
//    warp folds just those lanes' elements; otherwise (rare: one-signed or
//    degenerate blocks) one more pass over the block folds every unselected
//    element;
//  * fallback (blocks under 1024 entries, k > L/8, too few candidates after
//    the retry, or a dropped key at or above the threshold): exact radix
//    select on all keys by streaming passes over the block (it is in L2 by
//    then), 8 bits per pass, then one placing pass (ascending index order).
// HBM traffic per parameter: 2 B gradient + 0.5 B codes read; per selected
// entry 4 B written.
#include "mua_kernels.cuh"

// Warps (= blocks in flight) per CTA and candidate slots per lane, for blocks
// of up to 16384 entries (S) and up to 32768 entries (L).
#ifndef MUA_SELECT_WARPS_S
#define MUA_SELECT_WARPS_S 1
#endif
#ifndef MUA_SELECT_CAP_S
#define MUA_SELECT_CAP_S 32
#endif
#ifndef MUA_SELECT_MINB_S
#define MUA_SELECT_MINB_S (24 / MUA_SELECT_WARPS_S)  // up to 24 warps per SM (9 KB of shared memory each)
#endif
#ifndef MUA_SELECT_WARPS_L
#define MUA_SELECT_WARPS_L 4
#endif
#ifndef MUA_SELECT_MINB_L
#define MUA_SELECT_MINB_L 3
#endif
#ifndef MUA_SELECT_CAP_L
#define MUA_SELECT_CAP_L 48
#endif

namespace mua {
namespace {

constexpr uint32_t kFull = 0xFFFFFFFFu;
constexpr uint32_t kKeyInf = 0x7F800000u;  // key of +-inf; every threshold stays <= it
#ifndef MUA_SELECT_UNROLL
#define MUA_SELECT_UNROLL 1
#endif
constexpr int kUnroll = MUA_SELECT_UNROLL;  // 256-element steps per load group
// 256-element steps of a whole-step block that one lane asks L2 to fetch (a
// bulk prefetch, no completion to wait for) before the threshold sample, so
// the streaming pass finds them on chip. The default covers a 16384 block.
#ifndef MUA_SELECT_PREFETCH_STEPS
#define MUA_SELECT_PREFETCH_STEPS 64
#endif

// CAP: candidate slots per lane. A candidate takes 6 bytes (its a_t bits
// and its block index in two arrays).
template <int CAP>
struct WarpSmem {
  uint32_t ckey[CAP * 32];  // lane l's i-th candidate at [32 i + l]: bits of a_t
  uint16_t cidx[CAP * 32];  // ... and its block-relative index
  uint32_t hist[256];       // radix histogram
};

template <int CAP, int WARPS>
struct CtaSmem {
  WarpSmem<CAP> w[WARPS];
};

// The 16 dequantization levels of the step, one table per CTA. A namespace-
// scope array has a fixed shared address: every lookup is one load at a
// constant offset from the code's byte offset, in the out-of-line helpers too.
__shared__ float s_levels[16];

__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t x, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(kFull, x, o);
    if (lane >= o) x += y;
  }
  return x;
}

// One 256-element step: lane l holds elements e0 .. e0 + 7 of the block
// (gradient bits and packed codes; +0 and code 0 past L).
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

// a_t of element e of a step: f32(g) + level[code]. The code word is read as
// byte offsets into the level table (nibble * 4).
__device__ __forceinline__ float level_of(uint32_t cv, int e) {
  const uint32_t off = (e == 0) ? ((cv << 2) & 0x3Cu) : ((cv >> (4 * e - 2)) & 0x3Cu);
  return *reinterpret_cast<const float*>(reinterpret_cast<const char*>(s_levels) + off);
}
__device__ __forceinline__ float dequant1(const uint4& gv, uint32_t cv, int e) {
  return __fadd_rn(__uint_as_float(grad_bits(gv, e)), level_of(cv, e));
}
// Elements 2i and 2i + 1 with one paired add (the same two roundings).
__device__ __forceinline__ void dequant2(const uint4& gv, uint32_t cv, int i, float& a0, float& a1) {
  const uint32_t w = chunk_word(gv, i);
  const uint64_t g2 = ((uint64_t)(w & 0xFFFF0000u) << 32) | (uint32_t)(w << 16);
  const uint64_t a2 = f2_add_rn(g2, f2_pack(level_of(cv, 2 * i), level_of(cv, 2 * i + 1)));
  a0 = f2_lo(a2);
  a1 = f2_hi(a2);
}

// Bits of a_t for the 8 elements of a step, +0 past L.
__device__ __forceinline__ void dequant8(const uint4& gv, uint32_t cv, int e0, int L,
                                         uint32_t (&ab)[kChunk]) {
#pragma unroll
  for (int e = 0; e < kChunk; ++e) ab[e] = (e0 + e < L) ? __float_as_uint(dequant1(gv, cv, e)) : 0u;
}

// Shared-memory accesses of one candidate by the 32-bit shared-window
// addresses of its key and index slots (the 16-bit index moves through a
// 32-bit register, which PTX allows for narrow loads and stores) (the index slot sits at a fixed
// distance, half the key's offset, in its own array). The candidate regions are
// touched through these only, and a lane only ever touches its own region, so
// the volatile asm statements (kept in program order) are all the ordering
// they need. A candidate is read back as {key bits, index}, or as its key
// (|a| bits) alone.
__device__ __forceinline__ void sts_cand(uint32_t ka, uint32_t ia, uint32_t bits, uint32_t idx) {
  asm volatile("st.shared.b32 [%0], %2;\n st.shared.b16 [%1], %3;"
               ::"r"(ka), "r"(ia), "r"(bits), "r"(idx));
}
__device__ __forceinline__ uint32_t lds_key(uint32_t ka) {
  uint32_t k;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(k) : "r"(ka));
  return k & 0x7FFFFFFFu;
}
__device__ __forceinline__ uint2 lds_cand(uint32_t ka, uint32_t ia) {
  uint32_t k, i;
  asm volatile("ld.shared.b32 %0, [%2];\n ld.shared.u16 %1, [%3];"
               : "=r"(k), "=r"(i) : "r"(ka), "r"(ia));
  return make_uint2(k, i);
}

// Per-lane state of the candidate pass. The lane's region is key slots
// base + 128 i and index slots ibase + 64 i (the 32 lanes interleaved).
template <int CAP>
struct Lane {
  uint32_t slot;    // shared address of the next free key slot
  uint32_t islot;   // ... and of the next free index slot
  uint32_t base;    // shared address of the lane's first key slot
  uint32_t ibase;   // ... and of its first index slot
  uint32_t tau;     // candidate threshold key (>= the warp's tau_lo, <= kKeyInf)
  float tau_f;      // the same threshold as a float: |a| >= tau_f <=> key >= tau
  float rmin, rmax; // min / max of the entries make_room dropped
  __device__ __forceinline__ int count() const { return (int)((slot - base) >> 7); }
  __device__ __forceinline__ bool full() const { return slot > base + 128u * (CAP - kChunk); }
};

// Makes room in a lane's region for one more 8-element step: while it holds
// more than CAP - 8 entries, every entry with one of its two smallest keys is
// dropped into the residual's min/max (the others are compacted) and the
// lane's threshold rises above those keys, so every key the lane ever drops
// is below its final threshold. (Dropping two key values at a time halves
// the calls of a lane whose elements keep crossing its threshold.)
template <int CAP>
__device__ __noinline__ Lane<CAP> make_room(Lane<CAP> st, uint32_t* status) {
  while (st.full()) {
    const int n = st.count();
    uint32_t m0 = kFull;
    for (int i = 0; i < n; ++i)
      m0 = min(m0, lds_cand(st.base + 128u * i, st.ibase + 64u * i).x & 0x7FFFFFFFu);
    uint32_t m1 = kFull;  // the second smallest key, if any
    for (int i = 0; i < n; ++i) {
      const uint32_t key = lds_cand(st.base + 128u * i, st.ibase + 64u * i).x & 0x7FFFFFFFu;
      if (key > m0) m1 = min(m1, key);
    }
    if (m1 != kFull) m0 = m1;
    uint32_t kept = 0u;
    for (int i = 0; i < n; ++i) {
      const uint2 e = lds_cand(st.base + 128u * i, st.ibase + 64u * i);
      if ((e.x & 0x7FFFFFFFu) <= m0) {
        st.rmin = fminf(st.rmin, __uint_as_float(e.x));
        st.rmax = fmaxf(st.rmax, __uint_as_float(e.x));
      } else {
        sts_cand(st.base + 128u * kept, st.ibase + 64u * kept, e.x, e.y);
        ++kept;
      }
    }
    if (m0 >= kKeyInf) atomicOr(status, kStatusNonFinite);
    st.slot = st.base + 128u * kept;
    st.islot = st.ibase + 64u * kept;
    st.tau = max(st.tau, min(m0 + 1u, kKeyInf));
    st.tau_f = __uint_as_float(st.tau);
  }
  return st;
}

// Appends {bits of a, idx} at the lane's next slots and advances them iff
// |a| >= tau or a is NaN: one predicated compare, two stores and two adds, no
// branch.
__device__ __forceinline__ void append_if(uint32_t& slot, uint32_t& islot, float a, float tau,
                                          uint32_t idx) {
  asm volatile(
      "{\n"
      " .reg .pred p;\n"
      " .reg .f32 t;\n"
      " abs.f32 t, %2;\n"
      " setp.geu.f32 p, t, %3;\n"
      " @p st.shared.b32 [%0], %4;\n"
      " @p st.shared.b16 [%1], %5;\n"
      " @p add.u32 %0, %0, 128;\n"
      " @p add.u32 %1, %1, 64;\n"
      "}\n"
      : "+r"(slot), "+r"(islot)
      : "f"(a), "f"(tau), "r"(__float_as_uint(a)), "r"(idx));
}

// The streaming test of one step: every |a| >= the lane's threshold (NaN
// included) is appended. FULL: all 8 elements lie inside the block.
template <int CAP, bool FULL>
__device__ __forceinline__ void scan_step(const uint4& gv, uint32_t cv, int e0, int L,
                                          Lane<CAP>& st, uint32_t* status) {
  if (st.full()) st = make_room(st, status);
  float a[kChunk];
#pragma unroll
  for (int i = 0; i < kChunk / 2; ++i) dequant2(gv, cv, i, a[2 * i], a[2 * i + 1]);
#pragma unroll
  for (int e = 0; e < kChunk; ++e) {
    if (FULL || e0 + e < L) append_if(st.slot, st.islot, a[e], st.tau_f, (uint32_t)(e0 + e));
  }
}

// The candidate pass over a block with threshold tau_lo: full steps in
// groups of kUnroll, two groups of loads in flight, then the partial last
// step. Kept out of line: the retry calls it again.
template <bool VEC, int CAP>
__device__ __noinline__ Lane<CAP> stream_candidates(const StepArgs& A, int64_t start, int L,
                                                    uint32_t tau_lo,
                                                    uint32_t base, uint32_t ibase, int lane) {
  // The argument block is read once: after a call to make_room the compiler
  // would otherwise reload these from parameter space on every step.
  uint32_t* const status = &A.hdr[kHdrStatus];
  const uint16_t* const grads = A.grads;
  const uint8_t* const codes = A.codes;
  Lane<CAP> st;
  st.base = st.slot = base;
  st.ibase = st.islot = ibase;
  st.tau = tau_lo;
  st.tau_f = __uint_as_float(tau_lo);
  st.rmin = st.rmax = 0.0f;
  const int nfull = L >> 8;
  uint4 ga[kUnroll], gb[kUnroll];
  uint32_t ca[kUnroll], cb[kUnroll];
  if (VEC && (L & 255) == 0 && (nfull % (2 * kUnroll)) == 0) {
    // Whole 256-element steps in whole pairs of groups (every block of a
    // B_d = 16384 vector): lane pointers set once, compile-time offsets within
    // a group, no per-step bounds checks.
    const uint16_t* gp = grads + start + 8 * lane;
    const uint8_t* cp = codes + ((start + 8 * lane) >> 1);
    auto load_full = [&](uint4 (&g)[kUnroll], uint32_t (&c)[kUnroll], int s0) {
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        g[u] = ld_stream_v4(gp + 256 * (s0 + u));
        c[u] = ld_stream_u32(cp + 128 * (s0 + u));
      }
    };
    auto run_full = [&](const uint4 (&g)[kUnroll], const uint32_t (&c)[kUnroll], int s0) {
#pragma unroll
      for (int u = 0; u < kUnroll; ++u)
        scan_step<CAP, true>(g[u], c[u], ((s0 + u) << 8) + 8 * lane, L, st, status);
    };
    load_full(ga, ca, 0);
    for (int s0 = 0; s0 < nfull; s0 += 2 * kUnroll) {
      load_full(gb, cb, s0 + kUnroll);
      run_full(ga, ca, s0);
      if (s0 + 2 * kUnroll < nfull) load_full(ga, ca, s0 + 2 * kUnroll);
      run_full(gb, cb, s0 + kUnroll);
    }
    return st;
  }
  auto load_group = [&](uint4 (&g)[kUnroll], uint32_t (&c)[kUnroll], int s0) {
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
      if (s0 + u < nfull)
        load_step<VEC>(grads, codes, start, L, ((s0 + u) << 8) + 8 * lane, g[u], c[u]);
  };
  auto run_group = [&](const uint4 (&g)[kUnroll], const uint32_t (&c)[kUnroll], int s0) {
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
      if (s0 + u < nfull)
        scan_step<CAP, true>(g[u], c[u], ((s0 + u) << 8) + 8 * lane, L, st, status);
  };
  load_group(ga, ca, 0);
  for (int s0 = 0; s0 < nfull; s0 += 2 * kUnroll) {
    load_group(gb, cb, s0 + kUnroll);
    run_group(ga, ca, s0);
    load_group(ga, ca, s0 + 2 * kUnroll);
    run_group(gb, cb, s0 + kUnroll);
  }
  if ((nfull << 8) < L) {  // the block's partial last step
    const int e0 = (nfull << 8) + 8 * lane;
    uint4 gv;
    uint32_t cv;
    load_step<VEC>(grads, codes, start, L, e0, gv, cv);
    scan_step<CAP, false>(gv, cv, e0, L, st, status);
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
  uint32_t running = __shfl_sync(kFull, incl, 31) - incl;  // bins above this lane
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
  const int src = __ffs(__ballot_sync(kFull, found)) - 1;
  bin = __shfl_sync(kFull, fb, src & 31);
  above = __shfl_sync(kFull, fa, src & 31);
  inbin = __shfl_sync(kFull, fi, src & 31);
}

// Exact selection threshold among keys that all share the bits of `prefix`
// above bit hi (keys come from `for_each_key`, over the lane's entries). On
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

// The threshold sample: 64 chunks of 8 elements spread over the block (chunk
// c at element (c * (L / 64)) & ~7), each lane's two largest keys, sorted
// descending across the warp by a bitonic network (element r of the order in
// lane r / 2, slot r % 2). Returns the keys at rank `r` and at rank 63. The
// loads (sample_load) go out before the level table is ready.
template <bool VEC>
__device__ __forceinline__ void sample_load(const StepArgs& A, int64_t start, int L, int lane,
                                            uint4 (&gv)[2], uint32_t (&cv)[2]) {
  const int cstride = (L / 64) & ~7;
#pragma unroll
  for (int h = 0; h < 2; ++h)
    load_step<VEC>(A.grads, A.codes, start, L, (lane + 32 * h) * cstride, gv[h], cv[h]);
}
__device__ __forceinline__ void sample_threshold(const uint4 (&gv)[2], const uint32_t (&cv)[2],
                                                 int L, int r, int lane, uint32_t& tau_first,
                                                 uint32_t& tau_retry) {
  const int cstride = (L / 64) & ~7;
  uint32_t t1 = 0u, t2 = 0u;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int e0 = (lane + 32 * h) * cstride;
    uint32_t ab[kChunk];
    dequant8(gv[h], cv[h], e0, L, ab);
#pragma unroll
    for (int e = 0; e < kChunk; ++e) {
      const uint32_t key = ab[e] & 0x7FFFFFFFu;
      const uint32_t lo = min(t1, key);
      t1 = max(t1, key);
      t2 = max(t2, lo);
    }
  }
  uint32_t v0 = max(t1, t2), v1 = min(t1, t2);
#pragma unroll
  for (int size = 2; size <= 64; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const bool up = (((2 * lane) & size) == 0);
      if (stride == 1) {  // within the lane: elements 2 lane, 2 lane + 1
        const uint32_t hi2 = max(v0, v1), lo2 = min(v0, v1);
        v0 = up ? hi2 : lo2;
        v1 = up ? lo2 : hi2;
      } else {
        const int ls = stride >> 1;  // lane distance
        const uint32_t o0 = __shfl_xor_sync(kFull, v0, ls);
        const uint32_t o1 = __shfl_xor_sync(kFull, v1, ls);
        const bool keep_max = (((lane & ls) == 0) == up);
        v0 = keep_max ? max(v0, o0) : min(v0, o0);
        v1 = keep_max ? max(v1, o1) : min(v1, o1);
      }
    }
  }
  const uint32_t tl0 = __shfl_sync(kFull, v0, r >> 1);
  const uint32_t tl1 = __shfl_sync(kFull, v1, r >> 1);
  tau_first = min((r & 1) ? tl1 : tl0, kKeyInf);
  tau_retry = min(__shfl_sync(kFull, v1, 31), kKeyInf);  // the smallest of the 64
}

// Folds unselected elements into the lane's residual min/max: those of the
// lanes in `open` (each lane's eight-element chunk of every 256-element step,
// spread over the warp), or every element of the block when `open` is 0. An
// element is selected iff its key is above thr, or equals it with an index
// below its owner lane's `cut`.
template <bool VEC>
__device__ __noinline__ void fold_unselected(const StepArgs& A, int64_t start, int L,
                                             uint32_t thr, uint32_t cut, uint32_t open,
                                             int lane, float& rmin, float& rmax) {
  const int nsteps = (L + 255) >> 8;
  auto fold_step = [&](int e0, uint32_t c) {  // the unselected elements e0 .. e0 + 7
    uint4 gv;
    uint32_t cv;
    load_step<VEC>(A.grads, A.codes, start, L, e0, gv, cv);
    uint32_t ab[kChunk];
    dequant8(gv, cv, e0, L, ab);
#pragma unroll
    for (int e = 0; e < kChunk; ++e) {
      const uint32_t key = ab[e] & 0x7FFFFFFFu;
      if (e0 + e >= L || key > thr || (key == thr && (uint32_t)(e0 + e) < c)) continue;
      rmin = fminf(rmin, __uint_as_float(ab[e]));
      rmax = fmaxf(rmax, __uint_as_float(ab[e]));
    }
  };
  if (open == 0u) {
    for (int s = 0; s < nsteps; ++s) fold_step((s << 8) + 8 * lane, cut);
    return;
  }
  while (open) {
    const int l = __ffs(open) - 1;
    open &= open - 1;
    const uint32_t cl = __shfl_sync(kFull, cut, l);
    for (int s = lane; s < nsteps; s += 32) fold_step((s << 8) + 8 * l, cl);
  }
}

template <bool VEC, int LMAX, int CAP, int WARPS, int MINB>
__global__ void __launch_bounds__(WARPS * 32, MINB)
    mua_select_warp_kernel(const __grid_constant__ StepArgs A) {
  extern __shared__ __align__(16) uint8_t dyn[];
  CtaSmem<CAP, WARPS>& S = *reinterpret_cast<CtaSmem<CAP, WARPS>*>(dyn);
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const Geometry& G = A.g;
  const int j = blockIdx.x * WARPS + wid;
  const bool live = j < G.nb;
  int64_t start = 0;
  int L = 0;
  if (live) block_span(A, j, start, L);
  const int k = live ? block_k(G, L) : 0;
  const bool cand = live && L >= 1024 && L <= LMAX && 8 * k <= L;
  // The block's L2 prefetch and the threshold sample's loads go out first:
  // neither needs the level table.
  uint4 sg[2];
  uint32_t sc[2];
  if (cand) {
    if (VEC && (L & 255) == 0) {  // the streaming pass's data, on its way into L2
      const int n = min(MUA_SELECT_PREFETCH_STEPS, L >> 8);
      const bool pf = lane == 0 && aligned16(A.grads + start) && aligned16(A.codes + (start >> 1));
      prefetch_l2_if(pf, A.grads + start, 512u * n);
      prefetch_l2_if(pf, A.codes + (start >> 1), 128u * n);
    }
    sample_load<VEC>(A, start, L, lane, sg, sc);
  }
  {
    const float delta = 0.0f - __uint_as_float(A.hdr[A.pair_cur]);
    const float Delta = __uint_as_float(A.hdr[A.pair_cur + 1]);
    const float unit = __fdiv_rn(__fsub_rn(Delta, delta), 15.0f);
    fill_levels(s_levels, delta, unit);
  }
  __syncthreads();  // the only CTA barrier: the level table
  if (!live) return;
  WarpSmem<CAP>& W = S.w[wid];
  uint32_t* const status = &A.hdr[kHdrStatus];
  uint32_t* row = A.window + ((int64_t)j * G.m + A.row) * G.kp;
  const int nsteps = (L + 255) >> 8;

  float rmin = 0.0f, rmax = 0.0f;  // residual; selected entries become +0
  bool done = false;

  // ---------------- candidate path
  if (cand) {
    // rank of tau_lo among the 64 sampled values: ~2.5 % of the block above it
    const int r = min(63, (int)((1280u * (uint32_t)k + (uint32_t)L - 1u) / (uint32_t)L) - 1);
    uint32_t tau_first, tau_retry;
    sample_threshold(sg, sc, L, r, lane, tau_first, tau_retry);

    // One streaming pass per attempt (a second, with a lower tau_lo, only when
    // the first finds fewer than k candidates). An all-zero sample goes
    // straight to the fallback: every element would be a candidate.
    for (int attempt = 0; attempt < 2 && !done && tau_first != 0u; ++attempt) {
      const uint32_t tau_lo = attempt == 0 ? tau_first : tau_retry;
      if (attempt == 1 && tau_retry >= tau_first) break;
      const Lane<CAP> st = stream_candidates<VEC, CAP>(
          A, start, L, tau_lo, smem_addr(&W.ckey[lane]), smem_addr(&W.cidx[lane]), lane);
      const int mine = st.count();
      const uint32_t n = __reduce_add_sync(kFull, (uint32_t)mine);
      const uint32_t drop_bound = __reduce_max_sync(kFull, st.tau > tau_lo ? st.tau : 0u);
      const uint32_t T = __reduce_max_sync(kFull, st.tau);  // every non-candidate key < T
      if (n < (uint32_t)k) continue;  // too few: retry lower, else the fallback
      // the lane's i-th candidate: key slot cand + 128 i, index slot icand + 64 i
      const uint32_t cand = st.base, icand = st.ibase;
      auto entry = [&](int i) { return lds_cand(cand + 128u * i, icand + 64u * i); };
      auto key_of = [&](int i) { return lds_key(cand + 128u * i); };
      uint32_t kmax = 0u;
#pragma unroll 4
      for (int i = 0; i < mine; ++i) kmax = max(kmax, key_of(i));
      kmax = __reduce_max_sync(kFull, kmax);
      int mode = 1, need = k;
      uint32_t thr = tau_lo;
      const uint32_t diff = kmax ^ tau_lo;
      if (diff != 0u) {
        warp_radix(31 - __clz(diff), tau_lo, k, W.hist, lane,
                   [&](auto&& f) {
#pragma unroll 4
                     for (int i = 0; i < mine; ++i) f(key_of(i));
                   },
                   mode, thr, need);
      }
      // Exact only if every dropped key (< its lane's tau <= drop_bound) is below thr.
      if (drop_bound > thr) break;
      if (lane == 0 && kmax >= kKeyInf) atomicOr(status, kStatusNonFinite);
      // The selection: keys above thr, and keys equal to it (all of them in
      // mode 0; in mode 1 the `need` lowest indices over the warp). A lane's
      // entries ascend by index, so the ties a lane gives are a prefix of its
      // ties: those below `cut`, its first tie left out (0x10000: none).
      uint32_t cut = 0x10000u, won = 0u;
      if (mode == 1) {
        int cur = 0;
        auto next_tie = [&]() -> uint32_t {
          for (; cur < mine; ++cur) {
            const uint2 e = entry(cur);
            if ((e.x & 0x7FFFFFFFu) == thr) return e.y;
          }
          return 0x10000u;
        };
        uint32_t head = next_tie();
        for (int q = 0; q < need; ++q) {  // one tie per round: the lowest head
          if (head == __reduce_min_sync(kFull, head)) {
            ++won;
            ++cur;
            head = next_tie();
          }
        }
        cut = head;
      }
      // The row, lane by lane (each lane's entries in ascending index order):
      // a lane's first place is the count of entries the lanes below it give.
      uint32_t nsel = won;
#pragma unroll 4
      for (int i = 0; i < mine; ++i) {
        const uint32_t key = key_of(i);
        nsel += (key > thr || (mode == 0 && key == thr)) ? 1u : 0u;
      }
      uint32_t pos = warp_incl_scan(nsel, lane) - nsel;
      // Place the selected entries; the others join the residual's min/max.
      rmin = st.rmin;
      rmax = st.rmax;
      for (int i = 0; i < mine; ++i) {
        const uint2 e = entry(i);
        const uint32_t key = e.x & 0x7FFFFFFFu;
        if (key > thr || (key == thr && e.y < cut)) {
          put_row(row, pos, k, e.y, e.x);
          ++pos;
        } else {
          rmin = fminf(rmin, __uint_as_float(e.x));
          rmax = fmaxf(rmax, __uint_as_float(e.x));
        }
      }
      // Elements a lane never appended have |a| below that lane's final
      // threshold: tau_lo for lanes that never raised it. If the folded values
      // reach past +-tau_lo, only raised lanes whose threshold is beyond them
      // can still move the min or the max: their own elements are folded (two
      // steps per warp lane). Otherwise (rare: one-signed or degenerate blocks)
      // every unselected element of the block is.
      float bmin = rmin, bmax = rmax;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        bmin = fminf(bmin, __shfl_xor_sync(kFull, bmin, o));
        bmax = fmaxf(bmax, __shfl_xor_sync(kFull, bmax, o));
      }
      const float lo_f = __uint_as_float(tau_lo);
      if (bmax >= lo_f && bmin <= -lo_f) {
        const float mine_f = __uint_as_float(st.tau);
        const uint32_t open =
            __ballot_sync(kFull, st.tau > tau_lo && !(bmax >= mine_f && bmin <= -mine_f));
        if (open) fold_unselected<VEC>(A, start, L, thr, cut, open, lane, rmin, rmax);
      } else {
        fold_unselected<VEC>(A, start, L, thr, cut, 0u, lane, rmin, rmax);
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
        dequant8(gv, cv, e0, L, ab);
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
      dequant8(gv, cv, e0, L, ab);
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
      const uint32_t tot = __shfl_sync(kFull, incl, 31);
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
    kmax = __reduce_max_sync(kFull, kmax);
    if (lane == 0 && kmax >= kKeyInf) atomicOr(status, kStatusNonFinite);
  }

  for (int sl = k + lane; sl < G.kp; sl += 32) row[sl] = kEmptySlot;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    rmin = fminf(rmin, __shfl_xor_sync(kFull, rmin, o));
    rmax = fmaxf(rmax, __shfl_xor_sync(kFull, rmax, o));
  }
  if (lane == 0) {
    atomicMax(&A.hdr[A.pair_next], __float_as_uint(0.0f - rmin));  // >= +0, canonical zero
    atomicMax(&A.hdr[A.pair_next + 1], __float_as_uint(rmax + 0.0f));
  }
}

template <bool VEC, int LMAX, int CAP, int WARPS, int MINB>
cudaError_t launch_shape(const StepArgs& args, cudaStream_t stream) {
  auto kern = mua_select_warp_kernel<VEC, LMAX, CAP, WARPS, MINB>;
  const uint32_t smem = (uint32_t)sizeof(CtaSmem<CAP, WARPS>);
  static uint32_t opted[kMaxDevices] = {};
  const cudaError_t e = opt_in_smem(kern, smem, opted);
  if (e != cudaSuccess) return e;
  const int grid = (args.g.nb + WARPS - 1) / WARPS;
  kern<<<grid, WARPS * 32, smem, stream>>>(args);
  return cudaGetLastError();
}

}  // namespace

uint32_t select_warp_smem_bytes(int Bd) {
  return Bd <= 16384
             ? (uint32_t)sizeof(CtaSmem<MUA_SELECT_CAP_S, MUA_SELECT_WARPS_S>)
             : (uint32_t)sizeof(CtaSmem<MUA_SELECT_CAP_L, MUA_SELECT_WARPS_L>);
}

cudaError_t launch_select_warp(const StepArgs& args, bool vec, cudaStream_t stream) {
  if (args.g.Bd > 16384)
    return vec ? launch_shape<true, 32768, MUA_SELECT_CAP_L, MUA_SELECT_WARPS_L, MUA_SELECT_MINB_L>(
                     args, stream)
               : launch_shape<false, 32768, MUA_SELECT_CAP_L, MUA_SELECT_WARPS_L, MUA_SELECT_MINB_L>(
                     args, stream);
  return vec ? launch_shape<true, 16384, MUA_SELECT_CAP_S, MUA_SELECT_WARPS_S, MUA_SELECT_MINB_S>(
                   args, stream)
             : launch_shape<false, 16384, MUA_SELECT_CAP_S, MUA_SELECT_WARPS_S, MUA_SELECT_MINB_S>(
                   args, stream);
}

}  // namespace mua
