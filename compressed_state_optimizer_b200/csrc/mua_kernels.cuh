// Device-side building blocks of the two MicroAdam kernels (mua_select_warp.cu,
// mua_apply.cu) and the argument block both take.
//
// [MicroAdam ¶n] is paragraph n of "MicroAdam (Sparse-Gradient Adaptive
// Optimization with Quantized Error Feedback)".
//
// Element layout inside a block. A CTA of T threads owns one block of up to
// 32*T elements; thread `tid` holds 32 of them as 4 chunks of 8 consecutive
// elements, chunk c starting at block-local index c*8*T + 8*tid. So every
// chunk is one 16-byte load of bf16 gradients and one 4-byte load of packed
// codes, a warp's loads are contiguous, and the local index order is
// (c, tid, e) lexicographic, which the index-ordered scans rely on.
//
// Exact conversions without the (quarter-rate) conversion unit:
//   (float)c for 0 <= c < 2^23:  bits(0x4B000000 | c) - 2^23   (exact)
//   floor(x) for 0 <= x < 2^23:  bits(x + 2^23 rounded toward zero) - 0x4B000000
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

namespace mua {

constexpr int kElemsPerThread = 32;
constexpr int kChunk = 8;
constexpr int kChunks = kElemsPerThread / kChunk;
constexpr int kMaxWindow = 64;            // m <= 64 (ages fit a 6-bit field)
constexpr int kMaxSegments = 512;         // tensors of a list cut into blocks one by one
constexpr int kMaxWindowEntries = 15360;  // m * row_stride per block, on chip
constexpr uint32_t kEmptySlot = 0x0000FFFFu;  // I = -1, V = +0
constexpr uint32_t kNil = 0xFFFFFFFFu;

// Header words (uint32) at the start of the state buffer.
constexpr int kHdrPair0 = 0;   // (-delta, Delta) for even t
constexpr int kHdrPair1 = 2;   // (-delta, Delta) for odd t
constexpr int kHdrStatus = 4;
constexpr int kHdrBarrier = 5;  // arrivals at the fused kernel's grid barrier
constexpr uint32_t kStatusNonFinite = 1u;
constexpr uint32_t kStatusTimeout = 2u;  // a bounded wait gave up

struct Geometry {
  int64_t d;           // elements of this handle
  int64_t base_index;  // global index of element 0 (shards)
  int32_t Bd;          // block size B_d
  int32_t kb;          // k_b
  int32_t kp;          // window row stride (k_b rounded up to 4)
  int32_t m;           // window rows
  int32_t nb;          // blocks of this handle
  int32_t last_len;    // length of the last block
};

// One argument block for both kernels of step t.
struct StepArgs {
  Geometry g;
  float* params;       // fp32 parameters, or NULL when params16 is used
  uint16_t* params16;  // bf16 parameters (raw bits), or NULL
  const uint16_t* grads;
  uint8_t* codes;
  uint32_t* window;
  uint32_t* hdr;
  float* mhat;        // optional outputs (NULL in production)
  float* vhat;
  int32_t row;        // t mod m
  int32_t rows;       // min(t, m)
  int32_t pair_cur;   // header word of (-delta_t, Delta_t)
  int32_t pair_next;  // header word of (-delta_{t+1}, Delta_{t+1})
  uint32_t t_lo, t_hi;
  float lr, eps, decay, f1, f2;
  int32_t has_decay;
  uint32_t kp_recip;     // ceil(2^32 / kp): e / kp == __umulhi(e, kp_recip) for e < 2^16
  uint64_t wait_ns;      // longest wait at a grid barrier before giving up
  float w1[kMaxWindow];  // fp32(beta1^r), r = age
  float w2[kMaxWindow];  // fp32(beta2^r)
  uint32_t keys[10][2];  // Philox round keys: seed + r*(W0, W1)
  // Tensor lists cut per tensor (n_seg > 0): segment s holds elements
  // [seg_start[s], seg_start[s] + seg_len[s]) and blocks seg_first[s] ..
  // seg_first[s+1]-1 (a ragged last block each). n_seg == 0: the flat cut.
  int32_t n_seg;
  int32_t seg_first[kMaxSegments];
  int64_t seg_start[kMaxSegments];
  int64_t seg_len[kMaxSegments];
};

// Start (element offset within the handle) and length of block j. Kernels
// that call this take their StepArgs as a __grid_constant__ argument, so the
// indexed reads stay in the parameter bank.
// Entries a block of L parameters keeps: ceil(L k_b / B_d), k_b for a whole
// block (L k_b < 2^30 since B_d <= 32766, so 32-bit arithmetic is exact).
__device__ __forceinline__ int block_k(const Geometry& G, int L) {
  if (L == G.Bd) return G.kb;
  return (int)(((uint32_t)L * (uint32_t)G.kb + (uint32_t)G.Bd - 1u) / (uint32_t)G.Bd);
}

__device__ __forceinline__ void block_span(const StepArgs& A, int j, int64_t& start, int& L) {
  const Geometry& G = A.g;
  if (A.n_seg == 0) {
    start = (int64_t)j * G.Bd;
    L = (j == G.nb - 1) ? G.last_len : G.Bd;
    return;
  }
  int lo = 0, hi = A.n_seg - 1;  // the last segment whose first block is <= j
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (A.seg_first[mid] <= j) lo = mid; else hi = mid - 1;
  }
  const int64_t off = (int64_t)(j - A.seg_first[lo]) * G.Bd;
  start = A.seg_start[lo] + off;
  L = (int)min((int64_t)G.Bd, A.seg_len[lo] - off);
}

// ---------------------------------------------------------------- memory
// A 4-byte load with a 64-byte L2 fetch-size hint: the update's sparse
// parameter reads (a few per 128-byte line) then bring 64-byte halves from
// DRAM instead of whole lines (measured: 18 % fewer DRAM bytes read).
__device__ __forceinline__ float ld_sparse_f32(const float* p) {
  float v;
  asm volatile("ld.global.L2::64B.f32 %0, [%1];" : "=f"(v) : "l"(p));
  return v;
}
__device__ __forceinline__ float ld_sparse_bf16(const uint16_t* p) {
  uint16_t v;
  asm volatile("ld.global.L2::64B.u16 %0, [%1];" : "=h"(v) : "l"(p));
  return __uint_as_float((uint32_t)v << 16);
}

// Parameter storage: fp32, or bf16 rounded to nearest-even on every store.
template <bool BF16>
__device__ __forceinline__ float load_param_sparse(const StepArgs& A, int64_t i) {
  if constexpr (BF16) return ld_sparse_bf16(A.params16 + i);
  else return ld_sparse_f32(A.params + i);
}
template <bool BF16>
__device__ __forceinline__ float load_param(const StepArgs& A, int64_t i) {
  if constexpr (BF16) return __uint_as_float((uint32_t)A.params16[i] << 16);
  else return A.params[i];
}
template <bool BF16>
__device__ __forceinline__ void store_param(const StepArgs& A, int64_t i, float v) {
  if constexpr (BF16) A.params16[i] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
  else A.params[i] = v;
}

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}
__device__ __forceinline__ uint32_t ld_stream_u32(const void* p) {
  uint32_t v;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}
__device__ __forceinline__ bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// L2 prefetch hint for n bytes at p, issued only where `on` holds: no
// destination, no completion to wait for. p and n must be multiples of 16
// and the range must lie inside one allocation.
__device__ __forceinline__ void prefetch_l2_if(bool on, const void* p, uint32_t n) {
  asm volatile(
      "{\n"
      " .reg .pred q;\n"
      " setp.ne.b32 q, %2, 0;\n"
      " @q cp.async.bulk.prefetch.L2.global [%0], %1;\n"
      "}\n" ::"l"(p), "r"(n), "r"((uint32_t)on)
      : "memory");
}
// A 4-byte load of data this kernel also writes (the apply kernel's codes,
// which it overwrites in place): not through the read-only path.
__device__ __forceinline__ uint32_t ld_rw_u32(const void* p) {
  uint32_t v;
  asm volatile("ld.global.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}

// 32-bit shared-window address of a shared-memory object.
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

template <int T>
__device__ __forceinline__ int elem_index(int c, int tid, int e) {
  return c * kChunk * T + kChunk * tid + e;
}

// Loads the thread's 4 chunks: gradient bits as 4 words per chunk (word w holds
// elements 2w (low half) and 2w+1 (high half)), codes as one word per chunk
// (nibble e = element e). Elements at or past L read as g = +0, code = 0.
// The codes are read with coherent loads: the caller overwrites them.
// FULL (with VEC): all 32 T elements lie inside the block, no checks.
template <int T, bool VEC, bool FULL = false>
__device__ __forceinline__ void load_block(const uint16_t* __restrict__ grads,
                                           const uint8_t* __restrict__ codes, int64_t start,
                                           int L, int tid, uint4 (&gv)[kChunks],
                                           uint32_t (&cv)[kChunks]) {
#pragma unroll
  for (int c = 0; c < kChunks; ++c) {
    const int e0 = elem_index<T>(c, tid, 0);
    if ((VEC && FULL) || (VEC && e0 + kChunk <= L)) {
      gv[c] = ld_stream_v4(grads + start + e0);
      cv[c] = ld_rw_u32(codes + ((start + e0) >> 1));
    } else {
      uint32_t w[4] = {0u, 0u, 0u, 0u};
      uint32_t cw = 0u;
#pragma unroll
      for (int e = 0; e < kChunk; ++e) {
        if (e0 + e < L) {
          const int64_t i = start + e0 + e;
          const uint32_t gb = grads[i];
          const uint32_t byte = codes[i >> 1];
          const uint32_t nib = (i & 1) ? (byte >> 4) : (byte & 0xFu);
          w[e >> 1] |= gb << (16 * (e & 1));
          cw |= nib << (4 * e);
        }
      }
      gv[c] = make_uint4(w[0], w[1], w[2], w[3]);
      cv[c] = cw;
    }
  }
}

__device__ __forceinline__ uint32_t chunk_word(const uint4& v, int w) {
  return w == 0 ? v.x : (w == 1 ? v.y : (w == 2 ? v.z : v.w));
}

// fp32 bits of bf16 element e of a chunk.
__device__ __forceinline__ uint32_t grad_bits(const uint4& v, int e) {
  const uint32_t word = chunk_word(v, e >> 1);
  return (e & 1) ? (word & 0xFFFF0000u) : (word << 16);
}

// Two-wide fp32 arithmetic (sm_100 packed f32x2 instructions): each half is
// the IEEE operation with the stated rounding, bit for bit the scalar result;
// one instruction issues both. A pair is (low = x, high = y).
__device__ __forceinline__ uint64_t f2_pack(float x, float y) {
  return ((uint64_t)__float_as_uint(y) << 32) | __float_as_uint(x);
}
__device__ __forceinline__ float f2_lo(uint64_t v) { return __uint_as_float((uint32_t)v); }
__device__ __forceinline__ float f2_hi(uint64_t v) { return __uint_as_float((uint32_t)(v >> 32)); }
__device__ __forceinline__ uint64_t f2_add_rn(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_add_rz(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rz.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_sub_rn(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_mul_rn(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// Q^{-1} levels delta + c * unit for c = 0..15, each computed as
// fl(delta + fl(fl(c) * unit)) exactly as [MicroAdam ¶1]'s dequantization is
// written; threads 0..15 fill the table, the caller synchronizes.
__device__ __forceinline__ void fill_levels(float* lv, float delta, float unit) {
  const int c = threadIdx.x;
  if (c < 16) {
    const float cf = __fsub_rn(__uint_as_float(0x4B000000u | (uint32_t)c), 8388608.0f);
    lv[c] = __fadd_rn(delta, __fmul_rn(cf, unit));
  }
}

// One 4-bit code of stage (4): c = min(15, floor((floor(2^16 s) + r) / 2^16)),
// s16 = 2^16 s >= 0, r a 16-bit draw. Returns the code in bits 16..19 of the
// result (bits 0..15 are scratch); the caller shifts it into place.
__device__ __forceinline__ uint32_t quantize_code_hi(float s16, uint32_t r) {
  const uint32_t big = __float_as_uint(__fadd_rz(s16, 8388608.0f));  // 0x4B000000 + floor
  return __viaddmin_u32(big, r, 0x4B0FFFFFu);  // min(big + r, code 15)
}

// The fixed-point value `big` (below) of a = +0, the value every selected
// entry quantizes from: the same operations on the same operands.
__device__ __forceinline__ uint32_t quantize_big_zero(float dn, float inv16) {
  return __float_as_uint(__fadd_rz(__fmul_rn(__fsub_rn(0.0f, dn), inv16), 8388608.0f));
}

// Stage (4) for the 8 elements of a chunk [MicroAdam ¶1]: a2[i] holds the
// pair (a of element 2i, a of element 2i + 1) as fp32 bits (low, high);
// elements whose bit is set in `selbits` were selected and quantize as +0
// (their `big` is big0 = quantize_big_zero(delta, inv16)); x is the chunk's
// Philox4x32-10 output (element e draws the (e mod 2)-th 16-bit half of word
// e / 2); dn2 and inv2 hold (delta, delta) and (2^16 * 15 / (Delta - delta))
// twice. Returns the 8 codes packed into one word, element e in bits
// 4e .. 4e + 3.
//   s16 = (a - delta) * inv16, big = 2^23 + s16 rounded toward zero, so the low
//   mantissa of big is floor(s16); the code is min(15, (floor(s16) + r) >> 16),
//   which sits in bits 16..19 of min(big + r, 0x4B0FFFFF), i.e. in byte 2.
__device__ __forceinline__ uint32_t quantize8(const uint64_t (&a2)[4], uint32_t selbits,
                                              const uint4& x, uint64_t dn2, uint64_t inv2,
                                              uint32_t big0) {
  const uint64_t magic2 = f2_pack(8388608.0f, 8388608.0f);
  uint32_t hi[kChunk];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint64_t big2 = f2_add_rz(f2_mul_rn(f2_sub_rn(a2[i], dn2), inv2), magic2);
    const uint32_t b0 = ((selbits >> (2 * i)) & 1u) ? big0 : (uint32_t)big2;
    const uint32_t b1 = ((selbits >> (2 * i + 1)) & 1u) ? big0 : (uint32_t)(big2 >> 32);
    const uint32_t xw = chunk_word(x, i);
    hi[2 * i] = __viaddmin_u32(b0, xw & 0xFFFFu, 0x4B0FFFFFu);
    hi[2 * i + 1] = __viaddmin_u32(b1, xw >> 16, 0x4B0FFFFFu);
  }
  // Byte 2 of each (0..15, the code): even elements into one word, odd ones
  // into another, then one nibble interleave.
  const uint32_t ev = __byte_perm(__byte_perm(hi[0], hi[2], 0x0062u),
                                  __byte_perm(hi[4], hi[6], 0x0062u), 0x5410u);
  const uint32_t od = __byte_perm(__byte_perm(hi[1], hi[3], 0x0062u),
                                  __byte_perm(hi[5], hi[7], 0x0062u), 0x5410u);
  return ev | (od << 4);
}

// ---------------------------------------------------------------- scans
// Inclusive block scan with a single barrier: every warp re-scans the warp
// totals itself. `scratch` (T/32 entries) must not be written again before
// the next barrier.
template <int T, typename V>
__device__ __forceinline__ V block_scan_1bar(V x, V* scratch, V& total) {
  constexpr int NW = T / 32;
  const int lane = threadIdx.x & 31;
  const int wid = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const V y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  if constexpr (NW == 1) {
    total = __shfl_sync(0xFFFFFFFFu, x, 31);
    return x;
  } else {
    if (lane == 31) scratch[wid] = x;
    __syncthreads();
    V w = (lane < NW) ? scratch[lane] : V(0);
#pragma unroll
    for (int o = 1; o < NW; o <<= 1) {
      const V y = __shfl_up_sync(0xFFFFFFFFu, w, o);
      if (lane >= o) w += y;
    }
    const V off = __shfl_sync(0xFFFFFFFFu, w, (wid + 31) & 31);
    total = __shfl_sync(0xFFFFFFFFu, w, NW - 1);
    return x + (wid > 0 ? off : V(0));
  }
}

// ---------------------------------------------------------------- Philox
// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC'11) with precomputed round
// keys (keys[r] = the key bumped r times by the Weyl constants; the kernel
// argument block holds them, so each round's key is a constant-bank operand).
// Counter (c0, c1, c2, c3); returns the four output words.
__device__ __forceinline__ uint4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2,
                                               uint32_t c3, const uint32_t (&keys)[10][2]) {
  constexpr uint32_t M0 = 0xD2511F53u;
  constexpr uint32_t M1 = 0xCD9E8D57u;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint32_t hi0 = __umulhi(M0, c0), lo0 = M0 * c0;
    const uint32_t hi1 = __umulhi(M1, c2), lo1 = M1 * c2;
    const uint32_t n0 = hi1 ^ c1 ^ keys[r][0];
    const uint32_t n2 = hi0 ^ c3 ^ keys[r][1];
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
  }
  return make_uint4(c0, c1, c2, c3);
}

// Hardware approximations (PTX sqrt.approx / rcp.approx, relative error about
// 2^-22): the update's fp32 result is compared at 1e-5, far above that.
__device__ __forceinline__ float sqrt_approx(float x) {
  float r;
  asm("sqrt.approx.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// ---------------------------------------------------------------- AdamStats + update

// Asynchronous 16-byte global -> shared copies (cp.async, completed by the
// hardware; waiting on them is a wait_group, not a spin).
__device__ __forceinline__ void cp_async16(uint32_t dst_smem, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst_smem), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}

// Shared-memory layout of block_update (dynamic):
//   mask  u32[WnP]    bitmask of the window's index union (WnP = words padded to 4)
//   wpre  u16[WnP8]   exclusive popcount prefix of mask (union rank of each word)
//   W     u32[E]      staged rows, age-major; the index half becomes the union rank
//   acc   float2[Ucap] (sum_r beta1^r V_r, sum_r beta2^r V_r^2) per union slot
//   uidx  u16[Ucap]   block-relative index of each union slot
//   scan  u32[T/32]   block scan scratch
// Every region starts on a 16-byte boundary except uidx and scan (8 and 4).
__host__ __device__ inline int mask_words_padded(int Bd) { return (((Bd + 31) / 32) + 3) & ~3; }

__host__ __device__ inline uint32_t update_smem_bytes(int threads, int Bd, int kp, int m) {
  const int WnP = mask_words_padded(Bd);
  const int E = m * kp;
  const int Ucap = Bd < E ? Bd : E;
  return (uint32_t)(4 * WnP + 2 * ((WnP + 7) & ~7) + 4 * E + 10 * Ucap + 4 * (threads / 32));
}

// Byte offset of W (the staged rows) in block_update's shared memory.
__host__ __device__ inline uint32_t update_rows_offset(int Bd) {
  const int WnP = mask_words_padded(Bd);
  return (uint32_t)(4 * WnP + 2 * ((WnP + 7) & ~7));
}

// Starts copying block j's window rows of steps t, t-1, ..., t-rows+1 (age
// 0 first) into W, 16 bytes at a time: rows are kp = 4q entries long and
// start on 16-byte boundaries, so a copy never straddles two rows. The copies
// complete in the background; block_update waits for them. W must not be
// touched until then.
template <int T>
__device__ __forceinline__ void update_prefetch_rows(const StepArgs& A, int j, uint8_t* smem) {
  const Geometry& G = A.g;
  const uint32_t W = smem_addr(smem + update_rows_offset(G.Bd));
  const uint32_t* wblk = A.window + (int64_t)j * G.m * G.kp;
  const int staged4 = (A.rows * G.kp) >> 2;
  for (int v = threadIdx.x; v < staged4; v += T) {
    const int e = 4 * v;
    const int age = (int)__umulhi((uint32_t)e, A.kp_recip);
    int phys = A.row - age;
    if (phys < 0) phys += G.m;
    cp_async16(W + 16u * (uint32_t)v, wblk + phys * G.kp + (e - age * G.kp));
  }
}

// Stage (6) for block j [MicroAdam ¶1]: m_hat = AdamStats(beta1, G) and
// v_hat = AdamStats(beta2, G^2) over the block's window rows, then
// p <- p*(1 - lr*wd) - lr*m_hat/(eps + sqrt(v_hat)) on the window's index union
// and, if wd != 0, p <- p*(1 - lr*wd) on every other parameter of the block:
// each parameter is read and written once, and a bf16 parameter (BF16) is
// rounded once. The rows are staged in shared memory and a
// bitmask + popcount prefix gives each index its union rank. Two warps run
// the sums one row at a time, oldest row first: the indices of one row are
// distinct, so no two threads touch one accumulator within a row, and every
// accumulator sees its terms in the same order on every run. Called by all
// T threads, after a barrier.
template <int T, bool BF16>
__device__ __forceinline__ void block_update(const StepArgs& A, int j, int64_t start, int L,
                                             uint8_t* smem, const float* s_w1,
                                             const float* s_w2) {
  const int tid = threadIdx.x;
  const Geometry& G = A.g;
  const int Wn = (G.Bd + 31) >> 5;
  const int WnP = mask_words_padded(G.Bd);
  const int E = G.m * G.kp;
  const int Ucap = min(G.Bd, E);
  uint32_t* mask = reinterpret_cast<uint32_t*>(smem);
  uint16_t* wpre = reinterpret_cast<uint16_t*>(mask + WnP);
  uint32_t* W = reinterpret_cast<uint32_t*>(wpre + ((WnP + 7) & ~7));  // 16-byte aligned
  float2* acc = reinterpret_cast<float2*>(W + E);
  uint16_t* uidx = reinterpret_cast<uint16_t*>(acc + Ucap);
  uint32_t* scan = reinterpret_cast<uint32_t*>(uidx + Ucap);

  for (int w = tid; w < Wn; w += T) mask[w] = 0u;
  cp_async_wait_all();  // this thread's copies of the rows (update_prefetch_rows)
  __syncthreads();      // everyone's

  // The union of the staged rows' indices.
  const int staged4 = (A.rows * G.kp) >> 2;
  for (int v = tid; v < staged4; v += T) {
    const uint4 x = reinterpret_cast<const uint4*>(W)[v];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t idx = chunk_word(x, q) & 0xFFFFu;
      if (idx < (uint32_t)L) atomicOr(&mask[idx >> 5], 1u << (idx & 31));  // 0xFFFF: empty
    }
  }
  __syncthreads();

  // Union rank of each mask word (thread tid: words q tid .. q tid + q - 1).
  const int q = (Wn + T - 1) / T;
  uint32_t pc = 0u;
  for (int i = 0; i < q; ++i) {
    const int w = q * tid + i;
    if (w < Wn) pc += (uint32_t)__popc(mask[w]);
  }
  uint32_t U;
  uint32_t run = block_scan_1bar<T, uint32_t>(pc, scan, U) - pc;
  for (int i = 0; i < q; ++i) {
    const int w = q * tid + i;
    if (w < Wn) {
      wpre[w] = (uint16_t)run;
      run += (uint32_t)__popc(mask[w]);
    }
  }
  __syncthreads();

  // Each staged entry: index -> union rank (U <= 15360, so a rank never equals
  // the empty marker 0xFFFF); every slot's accumulator is cleared and its
  // index recorded (entries of one index write the same values).
  const int staged = A.rows * G.kp;
  for (int e = tid; e < staged; e += T) {
    const uint32_t v = W[e];
    const uint32_t idx = v & 0xFFFFu;
    if (idx >= (uint32_t)L) continue;
    const uint32_t w = idx >> 5;
    const uint32_t rank = wpre[w] + (uint32_t)__popc(mask[w] & ((1u << (idx & 31)) - 1u));
    W[e] = (v & 0xFFFF0000u) | rank;
    uidx[rank] = (uint16_t)idx;
    acc[rank] = make_float2(0.0f, 0.0f);
  }
  if (A.has_decay) {  // decay alone off the union (the union's comes with its update)
    for (int i = tid; i < L; i += T)
      if (!((mask[i >> 5] >> (i & 31)) & 1u))
        store_param<BF16>(A, start + i, __fmul_rn(load_param<BF16>(A, start + i), A.decay));
  }
  __syncthreads();

  // The parameters of this thread's first kPre union slots are loaded now,
  // so that their latency overlaps the sums.
  constexpr int kPre = 6;
  uint32_t pidx[kPre];
  float pv0[kPre];
#pragma unroll
  for (int b = 0; b < kPre; ++b) {
    const uint32_t r = (uint32_t)(b * T + tid);
    pidx[b] = (r < U) ? (uint32_t)uidx[r] : kNil;
    pv0[b] = (r < U) ? load_param_sparse<BF16>(A, start + pidx[b]) : 0.0f;
  }

  // The sums, one row at a time from the oldest: z <- z + beta^age * V.
  auto sum_row = [&](int age, int first, int stride) {
    const float c1 = s_w1[age], c2 = s_w2[age];
    const uint32_t* Wr = W + age * G.kp;
    for (int p = first; p < G.kp; p += stride) {
      const uint32_t v = Wr[p];
      const uint32_t r = v & 0xFFFFu;
      if (r == 0xFFFFu) continue;
      const float V = __uint_as_float(v & 0xFFFF0000u);
      float2 z = acc[r];
      z.x = __fadd_rn(z.x, __fmul_rn(c1, V));
      z.y = __fadd_rn(z.y, __fmul_rn(c2, __fmul_rn(V, V)));
      acc[r] = z;
    }
  };
  // Up to 16 rows, two warps do them with a 64-thread barrier between rows
  // (CTA-wide barriers cost the other warps more than the rows' work:
  // measured), and the CTA meets once after the last row; longer windows
  // spread each row over the whole CTA.
  constexpr int kSum = T < 64 ? T : 64;
  if (G.m <= 16) {
    if (tid < kSum) {
      for (int age = A.rows - 1; age >= 0; --age) {
        sum_row(age, tid, kSum);
        if constexpr (kSum == 32) {
          __syncwarp();
        } else {
          asm volatile("bar.sync 1, %0;" ::"n"(kSum) : "memory");  // the summing warps only
        }
      }
    }
    __syncthreads();
  } else {
    for (int age = A.rows - 1; age >= 0; --age) {
      sum_row(age, tid, T);
      __syncthreads();
    }
  }

  // Parameter update on the union: u = m_hat/(eps+sqrt(v_hat)) with the
  // hardware square root and reciprocal approximations (a few ulp, far inside
  // the fp32 update's error). First the preloaded slots, then the rest up to
  // kBatch slots per thread per round, all loads before any store.
  auto update_slot = [&](uint32_t r, uint32_t idx, float p) {
    const float2 z = acc[r];
    const float mh = __fmul_rn(A.f1, z.x);
    const float vh = __fmul_rn(A.f2, z.y);
    if (A.has_decay) p = __fmul_rn(p, A.decay);
    const float u = __fmul_rn(mh, rcp_approx(__fadd_rn(A.eps, sqrt_approx(vh))));
    store_param<BF16>(A, start + idx, __fsub_rn(p, __fmul_rn(A.lr, u)));
    if (A.mhat) {
      A.mhat[start + idx] = mh;
      A.vhat[start + idx] = vh;
    }
  };
#pragma unroll
  for (int b = 0; b < kPre; ++b)
    if (pidx[b] != kNil) update_slot((uint32_t)(b * T + tid), pidx[b], pv0[b]);
  constexpr int kBatch = 4;
  for (uint32_t r0 = kPre * T; r0 < U; r0 += kBatch * T) {
    uint32_t idx[kBatch];
    float pv[kBatch];
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const uint32_t r = r0 + (uint32_t)(b * T + tid);
      idx[b] = (r < U) ? (uint32_t)uidx[r] : kNil;
      pv[b] = (r < U) ? load_param_sparse<BF16>(A, start + idx[b]) : 0.0f;
    }
#pragma unroll
    for (int b = 0; b < kBatch; ++b)
      if (idx[b] != kNil) update_slot(r0 + (uint32_t)(b * T + tid), idx[b], pv[b]);
  }
}

// Copies the AdamStats weights into shared memory, one per thread (A must be
// the kernel's __grid_constant__ argument, so the indexed reads stay in the
// parameter bank). Caller synchronizes.
__device__ __forceinline__ void load_weights(const StepArgs& A, float* s_w1, float* s_w2) {
  for (int r = threadIdx.x; r < kMaxWindow; r += blockDim.x) {
    s_w1[r] = A.w1[r];
    s_w2[r] = A.w2[r];
  }
}

// ---------------------------------------------------------------- launchers
constexpr int kMaxDevices = 64;

// Raises a kernel's dynamic shared-memory limit to at least `smem` bytes, once
// per device and size: `opted` is the caller's record for that kernel (one
// static array per kernel instance). Devices past kMaxDevices opt in on every
// call.
template <typename Kern>
cudaError_t opt_in_smem(Kern kern, uint32_t smem, uint32_t (&opted)[kMaxDevices]) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool known = dev >= 0 && dev < kMaxDevices;
  if (known && opted[dev] >= smem) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess && known) opted[dev] = smem;
  return e;
}

// Host-side launchers (defined next to their kernels). Return a cudaError_t.
cudaError_t launch_apply(const StepArgs& args, int threads, bool vec, uint32_t smem,
                         cudaStream_t stream);  // bf16 parameters when args.params16
cudaError_t launch_select_warp(const StepArgs& args, bool vec, cudaStream_t stream);
uint32_t select_warp_smem_bytes(int Bd);
uint32_t apply_smem_bytes(int threads, int Bd, int kp, int m);
// The fused one-launch step (mua_fused.cu): how many of its CTAs the current
// device holds at once (0 if it cannot run this geometry), and its launch.
int fused_max_blocks(int Bd, int kp, int m, bool vec, bool bf16);
cudaError_t launch_fused(const StepArgs& args, bool vec, cudaStream_t stream);

}  // namespace mua
