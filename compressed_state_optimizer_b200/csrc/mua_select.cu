// Stage kernel 1 of the MicroAdam step ([MicroAdam ¶1] = paragraph 1 of
// "MicroAdam (Sparse-Gradient Adaptive Optimization with Quantized Error
// Feedback)"): for one block of B_d parameters per CTA,
//   a_t = g_t + Q^{-1}(e_t, delta_t, Delta_t)      (in registers, never stored)
//   (I_t, V_t) = Top-k of |a_t| (ties to the lower index), written in
//   ascending index order to row t mod m of the window G,
//   the residual (a_t with the selected entries zeroed) reduced to its block
//   min/max and folded into the global (-delta_{t+1}, Delta_{t+1}) pair with
//   one pair of integer atomics per CTA.
//
// Top-k is an exact MSB-first radix select on the 31-bit magnitude patterns
// (digits of 11, 11 and 9 bits, shared-memory histograms), followed by one
// index-ordered block scan that places the selected entries. HBM traffic per
// parameter: 2 B gradient + 0.5 B codes read; per selected entry 4 B written.
#include "mua_kernels.cuh"

namespace mua {
namespace {

constexpr int kHistBins = 2048;

// Finds the digit bin holding the krem-th largest remaining key: the largest b
// with (count of bins >= b) >= krem. Writes the bin and the count strictly
// above it to s_res[0], s_res[1].
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

template <int T, bool VEC>
__global__ void __launch_bounds__(T, (T <= 512 ? 1024 / T : 1)) mua_select_kernel(const SelectArgs A) {
  __shared__ uint32_t hist[kHistBins];
  __shared__ uint32_t scan32[T / 32];
  __shared__ unsigned long long scan64[2][T / 32];
  __shared__ uint32_t s_res[2];
  __shared__ float s_min[T / 32], s_max[T / 32];

  const int tid = threadIdx.x;
  const int j = blockIdx.x;
  const Geometry& G = A.g;
  const int64_t start = (int64_t)j * G.Bd;
  const int L = (j == G.nb - 1) ? G.last_len : G.Bd;
  const int k = (int)(((int64_t)L * G.kb + G.Bd - 1) / G.Bd);

  uint4 gv[kChunks];
  uint32_t cv[kChunks];
  load_block<T, VEC>(A.grads, A.codes, start, L, tid, gv, cv);

  // (1) a_t = g_t + Q^{-1}(e_t, delta_t, Delta_t).
  const float delta = 0.0f - __uint_as_float(A.hdr[A.pair_cur]);
  const float Delta = __uint_as_float(A.hdr[A.pair_cur + 1]);
  const float unit = __fdiv_rn(__fsub_rn(Delta, delta), 15.0f);
  float af[kElemsPerThread];
  dequant_block<T>(gv, cv, delta, unit, af);
  // Only the bit patterns stay live; the magnitude key is ab & 0x7FFFFFFF and
  // every radix digit below lies in bits 0..30, so it reads ab directly.
  uint32_t ab[kElemsPerThread];
#pragma unroll
  for (int i = 0; i < kElemsPerThread; ++i) ab[i] = __float_as_uint(af[i]);
  if (L < kElemsPerThread * T) {  // slots past the block's end hold +0
#pragma unroll
    for (int c = 0; c < kChunks; ++c)
#pragma unroll
      for (int e = 0; e < kChunk; ++e)
        if (elem_index<T>(c, tid, e) >= L) ab[c * kChunk + e] = 0u;
  }

  // (2) exact radix select of the k-th largest magnitude key tau.
  uint32_t prefix = 0u, pmask = 0u;
  int krem = k;
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 20 : (pass == 1 ? 9 : 0);
    const int nbins = pass == 2 ? 512 : kHistBins;
    for (int b = tid; b < nbins; b += T) hist[b] = 0u;
    if (tid == 0) {
      s_res[0] = 0u;
      s_res[1] = 0u;
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kElemsPerThread; ++i) {
      if ((ab[i] & pmask) == prefix) atomicAdd(&hist[(ab[i] >> shift) & (nbins - 1)], 1u);
    }
    __syncthreads();
    if (pass == 0 && tid == 0) {
      // Keys >= 0x7F800000 (bins 0x7F8..0x7FF) are +-inf or NaN.
      uint32_t bad = 0;
      for (int b = 0x7F8; b < kHistBins; ++b) bad |= hist[b];
      if (bad) atomicOr(&A.hdr[kHdrStatus], kStatusNonFinite);
    }
    find_bin<T>(hist, nbins, krem, scan32, s_res);
    __syncthreads();
    prefix |= s_res[0] << shift;
    pmask |= (uint32_t)(nbins - 1) << shift;
    krem -= (int)s_res[1];
    __syncthreads();
  }
  const uint32_t tau = prefix;
  const int need = krem;  // keys equal to tau to take, lowest indices first

  // Index-ordered positions: per chunk, counts of keys > tau and == tau,
  // packed in 16-bit fields (each field total <= 8*T <= 8192).
  unsigned long long pg = 0ull, pe = 0ull;
#pragma unroll
  for (int c = 0; c < kChunks; ++c) {
    uint32_t ng = 0, ne = 0;
#pragma unroll
    for (int e = 0; e < kChunk; ++e) {
      const uint32_t key = ab[c * kChunk + e] & 0x7FFFFFFFu;
      ng += key > tau;
      ne += key == tau;
    }
    pg |= (unsigned long long)ng << (16 * c);
    pe |= (unsigned long long)ne << (16 * c);
  }
  unsigned long long tg, te;
  const unsigned long long xg = block_inclusive_scan<T, unsigned long long>(pg, scan64[0], tg) - pg;
  const unsigned long long xe = block_inclusive_scan<T, unsigned long long>(pe, scan64[1], te) - pe;

  // (2)+(3) write the selected entries; the residual keeps the rest.
  uint32_t* row = A.window + ((int64_t)j * G.m + A.row) * G.kp;
  float rmin = 0.0f, rmax = 0.0f;  // selected entries become +0
  uint32_t base_g = 0, base_e = 0;
#pragma unroll
  for (int c = 0; c < kChunks; ++c) {
    uint32_t run_g = base_g + (uint32_t)((xg >> (16 * c)) & 0xFFFFu);
    uint32_t run_e = base_e + (uint32_t)((xe >> (16 * c)) & 0xFFFFu);
    base_g += (uint32_t)((tg >> (16 * c)) & 0xFFFFu);
    base_e += (uint32_t)((te >> (16 * c)) & 0xFFFFu);
#pragma unroll
    for (int e = 0; e < kChunk; ++e) {
      const float v = __uint_as_float(ab[c * kChunk + e]);
      const uint32_t key = ab[c * kChunk + e] & 0x7FFFFFFFu;
      bool sel = false;
      uint32_t pos = 0;
      if (key > tau) {
        sel = true;
        pos = run_g + min(run_e, (uint32_t)need);
        ++run_g;
      } else if (key == tau) {
        if (run_e < (uint32_t)need) {
          sel = true;
          pos = run_g + run_e;
        }
        ++run_e;
      }
      if (sel && pos < (uint32_t)k) {
        const uint32_t idx = (uint32_t)elem_index<T>(c, tid, e);
        const uint32_t vb = __bfloat16_as_ushort(__float2bfloat16_rn(v));
        row[pos] = (idx & 0xFFFFu) | (vb << 16);
      } else {
        rmin = fminf(rmin, v);
        rmax = fmaxf(rmax, v);
      }
    }
  }
  for (int s = k + tid; s < G.kp; s += T) row[s] = kEmptySlot;

  // (5 first half) block residual min/max -> global pair, as ordered uint32.
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    rmin = fminf(rmin, __shfl_xor_sync(0xFFFFFFFFu, rmin, o));
    rmax = fmaxf(rmax, __shfl_xor_sync(0xFFFFFFFFu, rmax, o));
  }
  if ((tid & 31) == 0) {
    s_min[tid >> 5] = rmin;
    s_max[tid >> 5] = rmax;
  }
  __syncthreads();
  if (tid == 0) {
    for (int w = 1; w < T / 32; ++w) {
      rmin = fminf(rmin, s_min[w]);
      rmax = fmaxf(rmax, s_max[w]);
    }
    const float negmin = 0.0f - rmin;  // >= +0, canonical zero
    const float maxv = rmax + 0.0f;    // >= +0
    atomicMax(&A.hdr[A.pair_next], __float_as_uint(negmin));
    atomicMax(&A.hdr[A.pair_next + 1], __float_as_uint(maxv));
  }
}

template <int T>
cudaError_t launch_t(const SelectArgs& args, bool vec, cudaStream_t stream) {
  if (vec)
    mua_select_kernel<T, true><<<args.g.nb, T, 0, stream>>>(args);
  else
    mua_select_kernel<T, false><<<args.g.nb, T, 0, stream>>>(args);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_select(const SelectArgs& args, int threads, bool vec, cudaStream_t stream) {
  switch (threads) {
    case 32: return launch_t<32>(args, vec, stream);
    case 64: return launch_t<64>(args, vec, stream);
    case 128: return launch_t<128>(args, vec, stream);
    case 256: return launch_t<256>(args, vec, stream);
    case 512: return launch_t<512>(args, vec, stream);
    case 1024: return launch_t<1024>(args, vec, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace mua
