// Device-side building blocks shared by the two MicroAdam kernels
// (mua_select.cu, mua_apply.cu) and the argument structs their launchers take.
//
// [MicroAdam ¶n] is paragraph n of "MicroAdam (Sparse-Gradient Adaptive
// Optimization with Quantized Error Feedback)".
//
// Element layout inside a block. A CTA of T threads owns one block of up to
// 32*T elements; thread `tid` holds 32 of them as 4 chunks of 8 consecutive
// elements, chunk c starting at block-local index c*8*T + 8*tid. So every
// chunk is one 16-byte load of bf16 gradients and one 4-byte load of packed
// codes, a warp's loads are contiguous, and the local index order is
// (c, tid, e) lexicographic, which the index-ordered scans below rely on.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

namespace mua {

constexpr int kElemsPerThread = 32;
constexpr int kChunk = 8;
constexpr int kChunks = kElemsPerThread / kChunk;
constexpr int kMaxWindow = 64;            // m <= 64 (ages fit a 6-bit field)
constexpr int kMaxWindowEntries = 16384;  // m * row_stride per block, on chip
constexpr uint32_t kEmptySlot = 0x0000FFFFu;  // I = -1, V = +0

// Header words (uint32) at the start of the state buffer.
constexpr int kHdrPair0 = 0;   // (-delta, Delta) for even t
constexpr int kHdrPair1 = 2;   // (-delta, Delta) for odd t
constexpr int kHdrStatus = 4;
constexpr uint32_t kStatusNonFinite = 1u;

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

struct SelectArgs {
  Geometry g;
  const uint16_t* grads;
  const uint8_t* codes;
  uint32_t* window;
  uint32_t* hdr;
  int32_t row;        // t mod m
  int32_t pair_cur;   // header word of (-delta_t, Delta_t)
  int32_t pair_next;  // header word of (-delta_{t+1}, Delta_{t+1})
};

struct ApplyArgs {
  Geometry g;
  float* params;
  const uint16_t* grads;
  uint8_t* codes;
  const uint32_t* window;
  uint32_t* hdr;
  float* mhat;
  float* vhat;
  int32_t row;        // t mod m
  int32_t rows;       // min(t, m)
  int32_t pair_cur;
  int32_t pair_next;
  uint32_t t_lo, t_hi;
  float lr, eps, decay, f1, f2;
  int32_t has_decay;
  int32_t reverse;     // process blocks in reverse order
  uint32_t smem_bytes;
  float w1[kMaxWindow];          // fp32(beta1^r), r = age
  float w2[kMaxWindow];          // fp32(beta2^r)
  uint32_t keys[10][2];          // Philox round keys: seed + r*(W0, W1)
};

// ---------------------------------------------------------------- memory
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

// Block-local element index of (chunk c, thread tid, element e).
template <int T>
__device__ __forceinline__ int elem_index(int c, int tid, int e) {
  return c * kChunk * T + kChunk * tid + e;
}

// Loads the thread's 4 chunks: gradient bits as 4 words per chunk (word w holds
// elements 2w (low half) and 2w+1 (high half)), codes as one word per chunk
// (nibble e = element e). Elements at or past L read as g = +0, code = 0.
template <int T, bool VEC>
__device__ __forceinline__ void load_block(const uint16_t* __restrict__ grads,
                                           const uint8_t* __restrict__ codes, int64_t start,
                                           int L, int tid, uint4 (&gv)[kChunks],
                                           uint32_t (&cv)[kChunks]) {
#pragma unroll
  for (int c = 0; c < kChunks; ++c) {
    const int e0 = elem_index<T>(c, tid, 0);
    if (VEC && e0 + kChunk <= L) {
      gv[c] = ld_stream_v4(grads + start + e0);
      cv[c] = ld_stream_u32(codes + ((start + e0) >> 1));
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

// a = f32(g) + (delta + f32(c) * unit), each operation rounded to nearest
// with no contraction: stage (1) of [MicroAdam ¶1], bit-identical in both
// kernels.
__device__ __forceinline__ float dequant_add(uint32_t gbits16, uint32_t code, float delta,
                                             float unit) {
  const float gf = __uint_as_float(gbits16 << 16);
  const float level = __fmul_rn(__uint2float_rn(code), unit);
  return __fadd_rn(gf, __fadd_rn(delta, level));
}

template <int T>
__device__ __forceinline__ void dequant_block(const uint4 (&gv)[kChunks],
                                              const uint32_t (&cv)[kChunks], float delta,
                                              float unit, float (&a)[kElemsPerThread]) {
#pragma unroll
  for (int c = 0; c < kChunks; ++c) {
#pragma unroll
    for (int e = 0; e < kChunk; ++e) {
      const uint32_t word = chunk_word(gv[c], e >> 1);
      const uint32_t gb = (e & 1) ? (word >> 16) : (word & 0xFFFFu);
      const uint32_t code = (cv[c] >> (4 * e)) & 0xFu;
      a[c * kChunk + e] = dequant_add(gb, code, delta, unit);
    }
  }
}

__device__ __forceinline__ uint32_t magnitude_key(float a) {
  return __float_as_uint(a) & 0x7FFFFFFFu;
}

// ---------------------------------------------------------------- scans
// Inclusive block scan over T threads (T a multiple of 32). `scratch` needs
// T/32 entries. Ends with a barrier so scratch can be reused at once.
template <int T, typename V>
__device__ __forceinline__ V block_inclusive_scan(V x, V* scratch, V& total) {
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
    if (wid == 0) {
      V w = (lane < NW) ? scratch[lane] : V(0);
#pragma unroll
      for (int o = 1; o < NW; o <<= 1) {
        const V y = __shfl_up_sync(0xFFFFFFFFu, w, o);
        if (lane >= o) w += y;
      }
      if (lane < NW) scratch[lane] = w;
    }
    __syncthreads();
    const V off = (wid > 0) ? scratch[wid - 1] : V(0);
    total = scratch[NW - 1];
    __syncthreads();
    return x + off;
  }
}

// ---------------------------------------------------------------- Philox
// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC'11) with precomputed round
// keys. Counter (c0, c1, c2, c3); returns the four output words.
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

// ---------------------------------------------------------------- launchers
// Host-side launchers (defined next to their kernels). Return a cudaError_t.
cudaError_t launch_select(const SelectArgs& args, int threads, bool vec, cudaStream_t stream);
cudaError_t launch_apply(const ApplyArgs& args, int threads, bool vec, cudaStream_t stream);
uint32_t apply_smem_bytes(int threads, int Bd, int kp, int m);

}  // namespace mua
