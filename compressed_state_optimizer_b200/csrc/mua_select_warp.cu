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
// barrier, and memory latency hides behind the other warps' blocks.
//
// Exact Top-k:
//  * candidate path (blocks of 1024 to 32 * MASKW entries, k <= L/8):
//    512 sample keys (64 chunks of 8 spread over the block), each lane's top
//    two, a warp sort of those 64 values -> tau_lo. One streaming pass (lane l
//    holds elements 256 s + 8 l .. + 7 of step s) tests each |a| against the
//    lane's threshold and appends the candidates {bits of a, index} to the
//    lane's own strided region with one predicated 8-byte store; nothing else
//    happens per element. A lane whose region fills drops its smallest keys
//    and raises its threshold above them (make_room). An exact warp radix
//    select over the candidates (8-bit digits from the highest bit where
//    tau_lo and the largest candidate differ) gives the k-th key; the result
//    is exact iff every raised lane threshold is at most that key (else the
//    block takes the fallback). The selected entries are marked in a bitmask
//    of the block (ties at the threshold by a lowest-index merge of the
//    lanes' regions), and a popcount prefix of the mask gives each its place
//    in the row;
//  * residual min/max without a per-element cost: every element that was not
//    appended has |a| below T, the largest lane threshold. The candidates that
//    were not selected (and the dropped ones) are folded into the block's min
//    and max; if that max is >= T and that min <= -T, no other element can
//    change them. Otherwise (rare: one-signed or degenerate blocks) one more
//    pass over the block folds every unselected element;
//  * fallback (blocks under 1024 entries, k > L/8, too few candidates after
//    the retry, or a dropped key at or above the threshold): exact radix
//    select on all keys by streaming passes over the block (it is in L2 by
//    then), 8 bits per pass, then one placing pass.
// HBM traffic per parameter: 2 B gradient + 0.5 B codes read; per selected
// entry 4 B written.
#include "mua_kernels.cuh"

// Warps (= blocks in flight) per CTA and candidate slots per lane, for blocks
// of up to 16384 entries (S) and up to 32768 entries (L).
#ifndef MUA_SELECT_WARPS_S
#define MUA_SELECT_WARPS_S 8
#endif
#ifndef MUA_SELECT_CAP_S
#define MUA_SELECT_CAP_S 32
#endif
#ifndef MUA_SELECT_MINB_S
#define MUA_SELECT_MINB_S (MUA_SELECT_WARPS_S == 8 ? 2 : 4)  // CTAs per SM its smem allows
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
#define MUA_SELECT_UNROLL 2
#endif
constexpr int kUnroll = MUA_SELECT_UNROLL;  // 256-element steps per load group

// MASKW: words of the selection bitmask, which covers one block (512 for
// blocks of up to 16384 entries, 1024 up to 32768). CAP: slots per lane.
template <int MASKW, int CAP>
struct WarpSmem {
  uint2 cand[CAP * 32];  // lane l's i-th candidate at [32 i + l]: {bits of a_t, index}
  uint32_t mask[MASKW];  // selection bitmask; its first 256 words are the radix histogram
  uint16_t wpre[MASKW];  // exclusive popcount prefix of the mask words
};

#ifndef MUA_SELECT_PAIR_TABLE
#define MUA_SELECT_PAIR_TABLE 0
#endif

template <int MASKW, int CAP, int WARPS>
struct CtaSmem {
  float levels[16];
#if MUA_SELECT_PAIR_TABLE
  float2 pairs[256];  // entry b: (level[b & 15], level[b >> 4]), one code byte
#endif
  WarpSmem<MASKW, CAP> w[WARPS];
};

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

__device__ __forceinline__ float lds_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}
#if MUA_SELECT_PAIR_TABLE
__device__ __forceinline__ float2 lds_f2(uint32_t addr) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr));
  return v;
}
#endif

// a_t of element e of a step: f32(g) + level[code]. The code word is read as
// byte offsets into the level table (nibble * 4).
__device__ __forceinline__ float dequant1(const uint4& gv, uint32_t cv, const float* lv, int e) {
  const char* lb = reinterpret_cast<const char*>(lv);
  const uint32_t off = (e == 0) ? ((cv << 2) & 0x3Cu) : ((cv >> (4 * e - 2)) & 0x3Cu);
  return __fadd_rn(__uint_as_float(grad_bits(gv, e)), *reinterpret_cast<const float*>(lb + off));
}
// The same with the level table given by its shared-window address (for code
// outside the kernel body, where a generic pointer would not be known to
// point into shared memory).
__device__ __forceinline__ float dequant1_sa(const uint4& gv, uint32_t cv, uint32_t lv_sa, int e) {
  const uint32_t off = (e == 0) ? ((cv << 2) & 0x3Cu) : ((cv >> (4 * e - 2)) & 0x3Cu);
  return __fadd_rn(__uint_as_float(grad_bits(gv, e)), lds_f32(lv_sa + off));
}

// Bits of a_t for the 8 elements of a step, +0 past L.
__device__ __forceinline__ void dequant8(const uint4& gv, uint32_t cv, const float* lv, int e0,
                                         int L, uint32_t (&ab)[kChunk]) {
#pragma unroll
  for (int e = 0; e < kChunk; ++e)
    ab[e] = (e0 + e < L) ? __float_as_uint(dequant1(gv, cv, lv, e)) : 0u;
}

// Shared-memory accesses of one candidate slot by its 32-bit shared-window
// address. The candidate regions are touched through these two only, and a
// lane only ever touches its own region, so the volatile asm statements (kept
// in program order) are all the ordering they need.
__device__ __forceinline__ void sts_u2(uint32_t addr, uint32_t x, uint32_t y) {
  asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(addr), "r"(x), "r"(y));
}
__device__ __forceinline__ uint2 lds_u2(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}

// Per-lane state of the candidate pass. The lane's region is slots
// base + 256 i (8-byte slots, the 32 lanes interleaved).
template <int CAP>
struct Lane {
  uint32_t slot;    // shared address of the next free slot
  uint32_t base;    // shared address of the lane's first slot
  uint32_t tau;     // candidate threshold key (>= the warp's tau_lo, <= kKeyInf)
  float tau_f;      // the same threshold as a float: |a| >= tau_f <=> key >= tau
  float rmin, rmax; // min / max of the entries make_room dropped
  __device__ __forceinline__ int count() const { return (int)((slot - base) >> 8); }
  __device__ __forceinline__ bool full() const { return slot > base + 256u * (CAP - kChunk); }
};

// Makes room in a lane's region for one more 8-element step: while it holds
// more than CAP - 8 entries, every entry with the smallest key is dropped into
// the residual's min/max (the others are compacted) and the lane's threshold
// rises above that key, so every key the lane ever drops is below its final
// threshold.
template <int CAP>
__device__ __noinline__ Lane<CAP> make_room(Lane<CAP> st, uint32_t* status) {
  while (st.full()) {
    const int n = st.count();
    uint32_t m0 = kFull;
    for (int i = 0; i < n; ++i) m0 = min(m0, lds_u2(st.base + 256u * i).x & 0x7FFFFFFFu);
    uint32_t kept = st.base;
    for (int i = 0; i < n; ++i) {
      const uint2 e = lds_u2(st.base + 256u * i);
      if ((e.x & 0x7FFFFFFFu) == m0) {
        st.rmin = fminf(st.rmin, __uint_as_float(e.x));
        st.rmax = fmaxf(st.rmax, __uint_as_float(e.x));
      } else {
        sts_u2(kept, e.x, e.y);
        kept += 256u;
      }
    }
    if (m0 >= kKeyInf) atomicOr(status, kStatusNonFinite);
    st.slot = kept;
    st.tau = max(st.tau, min(m0 + 1u, kKeyInf));
    st.tau_f = __uint_as_float(st.tau);
  }
  return st;
}

// Appends {bits of a, idx} at `slot` and advances it by one slot (256 bytes)
// iff |a| >= tau or a is NaN: one predicated compare, store and add, no branch.
__device__ __forceinline__ void append_if(uint32_t& slot, float a, float tau, uint32_t idx) {
  asm volatile(
      "{\n"
      " .reg .pred p;\n"
      " .reg .f32 t;\n"
      " abs.f32 t, %1;\n"
      " setp.geu.f32 p, t, %2;\n"
      " @p st.shared.v2.b32 [%0], {%3, %4};\n"
      " @p add.u32 %0, %0, 256;\n"
      "}\n"
      : "+r"(slot)
      : "f"(a), "f"(tau), "r"(__float_as_uint(a)), "r"(idx));
}

// The streaming test of one step: every |a| >= the lane's threshold (NaN
// included) is appended. FULL: all 8 elements lie inside the block.
template <int CAP, bool FULL>
__device__ __forceinline__ void scan_step(const uint4& gv, uint32_t cv, uint32_t lv_sa, int e0,
                                          int L, Lane<CAP>& st, uint32_t* status) {
  if (st.full()) st = make_room(st, status);
  float a[kChunk];
#if MUA_SELECT_PAIR_TABLE
  // lv_sa is the pair table: one 8-byte load per code byte (two elements)
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t off = (i == 0) ? ((cv << 3) & 0x7F8u) : ((cv >> (8 * i - 3)) & 0x7F8u);
    const float2 lev = lds_f2(lv_sa + off);
    const uint32_t w = chunk_word(gv, i);
    a[2 * i] = __fadd_rn(__uint_as_float(w << 16), lev.x);
    a[2 * i + 1] = __fadd_rn(__uint_as_float(w & 0xFFFF0000u), lev.y);
  }
#else
#pragma unroll
  for (int e = 0; e < kChunk; ++e) a[e] = dequant1_sa(gv, cv, lv_sa, e);
#endif
#pragma unroll
  for (int e = 0; e < kChunk; ++e) {
    if (FULL || e0 + e < L) append_if(st.slot, a[e], st.tau_f, (uint32_t)(e0 + e));
  }
}

// The candidate pass over a block with threshold tau_lo: full steps in
// groups of kUnroll, two groups of loads in flight, then the partial last
// step. Kept out of line: the retry calls it again.
template <bool VEC, int CAP>
__device__ __noinline__ Lane<CAP> stream_candidates(const StepArgs& A, int64_t start, int L,
                                                    uint32_t lv_sa, uint32_t tau_lo,
                                                    uint32_t base, int lane) {
  // The argument block is read once: after a call to make_room the compiler
  // would otherwise reload these from parameter space on every step.
  uint32_t* const status = &A.hdr[kHdrStatus];
  const uint16_t* const grads = A.grads;
  const uint8_t* const codes = A.codes;
  Lane<CAP> st;
  st.base = st.slot = base;
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
        scan_step<CAP, true>(g[u], c[u], lv_sa, ((s0 + u) << 8) + 8 * lane, L, st, status);
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
        scan_step<CAP, true>(g[u], c[u], lv_sa, ((s0 + u) << 8) + 8 * lane, L, st, status);
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
    scan_step<CAP, false>(gv, cv, lv_sa, e0, L, st, status);
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
// lane r / 2, slot r % 2). Returns the keys at rank `r` and at rank 63.
template <bool VEC>
__device__ __forceinline__ void sample_threshold(const StepArgs& A, int64_t start, int L,
                                                 const float* lv, int r, int lane,
                                                 uint32_t& tau_first, uint32_t& tau_retry) {
  const int cstride = (L / 64) & ~7;
  uint32_t t1 = 0u, t2 = 0u;
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

template <bool VEC, int MASKW, int CAP, int WARPS, int MINB>
__global__ void __launch_bounds__(WARPS * 32, MINB)
    mua_select_warp_kernel(const __grid_constant__ StepArgs A) {
  extern __shared__ __align__(16) uint8_t dyn[];
  CtaSmem<MASKW, CAP, WARPS>& S = *reinterpret_cast<CtaSmem<MASKW, CAP, WARPS>*>(dyn);
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const Geometry& G = A.g;
  {
    const float delta = 0.0f - __uint_as_float(A.hdr[A.pair_cur]);
    const float Delta = __uint_as_float(A.hdr[A.pair_cur + 1]);
    const float unit = __fdiv_rn(__fsub_rn(Delta, delta), 15.0f);
    fill_levels(S.levels, delta, unit);
#if MUA_SELECT_PAIR_TABLE
    for (int b = threadIdx.x; b < 256; b += WARPS * 32) {
      const float c0 = __fsub_rn(__uint_as_float(0x4B000000u | (uint32_t)(b & 15)), 8388608.0f);
      const float c1 = __fsub_rn(__uint_as_float(0x4B000000u | (uint32_t)(b >> 4)), 8388608.0f);
      S.pairs[b] = make_float2(__fadd_rn(delta, __fmul_rn(c0, unit)),
                               __fadd_rn(delta, __fmul_rn(c1, unit)));
    }
#endif
  }
  __syncthreads();  // the only CTA barrier: the level tables
  const int j = blockIdx.x * WARPS + wid;
  if (j >= G.nb) return;
  WarpSmem<MASKW, CAP>& W = S.w[wid];
  const float* lv = S.levels;
  uint32_t* const status = &A.hdr[kHdrStatus];
  int64_t start;
  int L;
  block_span(A, j, start, L);
  const int k = (int)(((int64_t)L * G.kb + G.Bd - 1) / G.Bd);
  uint32_t* row = A.window + ((int64_t)j * G.m + A.row) * G.kp;
  const int nsteps = (L + 255) >> 8;
  const int wn = (L + 31) >> 5;  // mask words of the block

  float rmin = 0.0f, rmax = 0.0f;  // residual; selected entries become +0
  bool done = false;

  // ---------------- candidate path
  if (L >= 1024 && L <= 32 * MASKW && 8 * k <= L) {
    // rank of tau_lo among the 64 sampled values: ~2.5 % of the block above it
    const int r = min(63, (int)((1280 * (int64_t)k + L - 1) / L) - 1);
    uint32_t tau_first, tau_retry;
    sample_threshold<VEC>(A, start, L, lv, r, lane, tau_first, tau_retry);

    // One streaming pass per attempt (a second, with a lower tau_lo, only when
    // the first finds fewer than k candidates). An all-zero sample goes
    // straight to the fallback: every element would be a candidate.
    for (int attempt = 0; attempt < 2 && !done && tau_first != 0u; ++attempt) {
      const uint32_t tau_lo = attempt == 0 ? tau_first : tau_retry;
      if (attempt == 1 && tau_retry >= tau_first) break;
#if MUA_SELECT_PAIR_TABLE
      const uint32_t stream_lv = smem_addr(S.pairs);
#else
      const uint32_t stream_lv = smem_addr(S.levels);
#endif
      const Lane<CAP> st = stream_candidates<VEC, CAP>(A, start, L, stream_lv, tau_lo,
                                                       smem_addr(&W.cand[lane]), lane);
      const int mine = st.count();
      const uint32_t n = __reduce_add_sync(kFull, (uint32_t)mine);
      const uint32_t drop_bound = __reduce_max_sync(kFull, st.tau > tau_lo ? st.tau : 0u);
      const uint32_t T = __reduce_max_sync(kFull, st.tau);  // every non-candidate key < T
      if (n < (uint32_t)k) continue;  // too few: retry lower, else the fallback
      const uint32_t cand = st.base;  // the lane's i-th candidate at cand + 256 i
      uint32_t kmax = 0u;
      for (int i = 0; i < mine; ++i) kmax = max(kmax, lds_u2(cand + 256u * i).x & 0x7FFFFFFFu);
      kmax = __reduce_max_sync(kFull, kmax);
      int mode = 1, need = k;
      uint32_t thr = tau_lo;
      const uint32_t diff = kmax ^ tau_lo;
      if (diff != 0u) {
        warp_radix(31 - __clz(diff), tau_lo, k, W.mask, lane,
                   [&](auto&& f) {
                     for (int i = 0; i < mine; ++i) f(lds_u2(cand + 256u * i).x & 0x7FFFFFFFu);
                   },
                   mode, thr, need);
      }
      // Exact only if every dropped key (< its lane's tau <= drop_bound) is below thr.
      if (drop_bound > thr) break;
      if (lane == 0 && kmax >= kKeyInf) atomicOr(status, kStatusNonFinite);
      // Selection bitmask: keys above the threshold (at or above it in mode 0) ...
      for (int w = lane; w < wn; w += 32) W.mask[w] = 0u;
      __syncwarp();
      for (int i = 0; i < mine; ++i) {
        const uint2 e = lds_u2(cand + 256u * i);
        const uint32_t key = e.x & 0x7FFFFFFFu;
        if (mode == 0 ? key >= thr : key > thr) atomicOr(&W.mask[e.y >> 5], 1u << (e.y & 31));
      }
      // ... and, in mode 1, the `need` lowest indices among keys equal to it,
      // one per round: the lowest unmarked tied index over all lanes.
      if (mode == 1) {
        for (int q = 0; q < need; ++q) {
          __syncwarp();
          uint32_t head = 0xFFFFu;
          for (int i = 0; i < mine; ++i) {
            const uint2 e = lds_u2(cand + 256u * i);
            if ((e.x & 0x7FFFFFFFu) != thr) continue;
            if (e.y < head && !((W.mask[e.y >> 5] >> (e.y & 31)) & 1u)) head = e.y;
          }
          const uint32_t low = __reduce_min_sync(kFull, head);
          if (head == low && head != 0xFFFFu) atomicOr(&W.mask[head >> 5], 1u << (head & 31));
        }
      }
      __syncwarp();
      // u16 exclusive popcount prefix of the mask words (lane l: words
      // MASKW/32 l ..)
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
            W.wpre[w0 + w] = (uint16_t)run;
            run += (uint32_t)__popc(W.mask[w0 + w]);
          }
        }
      }
      __syncwarp();
      // Place the selected entries; the others join the residual's min/max.
      rmin = st.rmin;
      rmax = st.rmax;
      for (int i = 0; i < mine; ++i) {
        const uint2 e = lds_u2(cand + 256u * i);
        const uint32_t word = W.mask[e.y >> 5];
        if ((word >> (e.y & 31)) & 1u) {
          const uint32_t pos = W.wpre[e.y >> 5] + (uint32_t)__popc(word & ((1u << (e.y & 31)) - 1u));
          put_row(row, pos, k, e.y, e.x);
        } else {
          rmin = fminf(rmin, __uint_as_float(e.x));
          rmax = fmaxf(rmax, __uint_as_float(e.x));
        }
      }
      // Elements never appended have |a| < T: they can only move the min or
      // the max if the folded values do not reach past +-T.
      const float Tf = __uint_as_float(T);
      float bmin = rmin, bmax = rmax;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        bmin = fminf(bmin, __shfl_xor_sync(kFull, bmin, o));
        bmax = fmaxf(bmax, __shfl_xor_sync(kFull, bmax, o));
      }
      if (!(bmax >= Tf && bmin <= -Tf)) {
        // One more pass: every unselected element of the block.
        for (int s = 0; s < nsteps; ++s) {
          const int e0 = (s << 8) + 8 * lane;
          uint4 gv;
          uint32_t cv;
          load_step<VEC>(A.grads, A.codes, start, L, e0, gv, cv);
          uint32_t ab[kChunk];
          dequant8(gv, cv, lv, e0, L, ab);
          const uint32_t sel = (e0 < L) ? (W.mask[e0 >> 5] >> (e0 & 31)) : 0xFFu;
#pragma unroll
          for (int e = 0; e < kChunk; ++e) {
            if (e0 + e >= L || ((sel >> e) & 1u)) continue;
            rmin = fminf(rmin, __uint_as_float(ab[e]));
            rmax = fmaxf(rmax, __uint_as_float(ab[e]));
          }
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
    warp_radix(30, 0u, k, W.mask, lane, stream_keys, mode, thr, need);
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

template <bool VEC, int MASKW, int CAP, int WARPS, int MINB>
cudaError_t launch_shape(const StepArgs& args, cudaStream_t stream) {
  auto kern = mua_select_warp_kernel<VEC, MASKW, CAP, WARPS, MINB>;
  const uint32_t smem = (uint32_t)sizeof(CtaSmem<MASKW, CAP, WARPS>);
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
             ? (uint32_t)sizeof(CtaSmem<512, MUA_SELECT_CAP_S, MUA_SELECT_WARPS_S>)
             : (uint32_t)sizeof(CtaSmem<1024, MUA_SELECT_CAP_L, MUA_SELECT_WARPS_L>);
}

cudaError_t launch_select_warp(const StepArgs& args, bool vec, cudaStream_t stream) {
  if (args.g.Bd > 16384)
    return vec ? launch_shape<true, 1024, MUA_SELECT_CAP_L, MUA_SELECT_WARPS_L, MUA_SELECT_MINB_L>(
                     args, stream)
               : launch_shape<false, 1024, MUA_SELECT_CAP_L, MUA_SELECT_WARPS_L, MUA_SELECT_MINB_L>(
                     args, stream);
  return vec ? launch_shape<true, 512, MUA_SELECT_CAP_S, MUA_SELECT_WARPS_S, MUA_SELECT_MINB_S>(
                   args, stream)
             : launch_shape<false, 512, MUA_SELECT_CAP_S, MUA_SELECT_WARPS_S, MUA_SELECT_MINB_S>(
                   args, stream);
}

}  // namespace mua
