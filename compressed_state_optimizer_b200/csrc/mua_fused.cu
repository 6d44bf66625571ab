// The whole MicroAdam step in ONE launch for vectors whose blocks can all be
// resident at once ([MicroAdam ¶1] = paragraph 1 of "MicroAdam
// (Sparse-Gradient Adaptive Optimization with Quantized Error Feedback)").
//
// One CTA of 512 threads per block, all CTAs resident (cooperative launch):
//   1. a_t = g_t + Q^{-1}(e_t, delta_t, Delta_t), 32 values per thread, kept
//      in registers for the whole step;
//   2. the block's Top-k by an exact radix select over those registers (11-,
//      10- and 10-bit digits of |a| with a shared histogram; ties to the lower
//      index), the row t mod m of G written in index order;
//   3. the residual's block min/max folded into the global (-delta_{t+1},
//      Delta_{t+1}) pair;
//   4. a grid-wide barrier: delta_{t+1} / Delta_{t+1} depend on every block;
//   5. e_{t+1} = Q(residual, delta_{t+1}, Delta_{t+1}) straight from the
//      registers (no second read of g_t and e_t), then the AdamStats update of
//      the block (block_update, as in the apply kernel).
// The arithmetic is that of the two-kernel path (same level table, same
// quantize8, same block_update), so both give the same bytes.
//
// The barrier counts arrivals in a header word of the state, which the host
// zeroes before the launch. Its wait is bounded by the global nanosecond
// timer: a CTA that waits longer than the handle's limit sets
// MUA_STATUS_TIMEOUT in the status word, skips the rest of the step and
// returns (that step's results are then unspecified); it never spins on.
#include "mua_kernels.cuh"

namespace mua {
namespace {

constexpr int kFusedThreads = 512;
constexpr int kFusedElems = kElemsPerThread * kFusedThreads;  // 16384
constexpr uint32_t kKeyInf = 0x7F800000u;

struct FusedShared {
  float levels[16];
  float w1[kMaxWindow], w2[kMaxWindow];
  uint32_t scan[32];
  uint32_t res[3];  // digit bin, keys in higher bins, keys in the bin
  float mn[32], mx[32];
  uint32_t km[32];
  uint32_t go;      // 1 once the grid barrier passed
};

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// One radix digit: the bin (of `nbins` counts in hist) holding the krem-th
// largest key. Thread t owns bins [t per, t per + per). Result in S.res.
template <int T>
__device__ __forceinline__ void find_bin(const uint32_t* hist, int nbins, int krem,
                                         FusedShared& S) {
  const int per = nbins / T;
  const int b0 = threadIdx.x * per;
  uint32_t own = 0;
  for (int b = 0; b < per; ++b) own += hist[b0 + b];
  uint32_t total;
  const uint32_t incl = block_scan_1bar<T, uint32_t>(own, S.scan, total);
  uint32_t running = total - incl;  // keys in bins above this thread's range
  for (int b = per - 1; b >= 0; --b) {
    const uint32_t h = hist[b0 + b];
    if (running < (uint32_t)krem && running + h >= (uint32_t)krem) {
      S.res[0] = (uint32_t)(b0 + b);
      S.res[1] = running;
      S.res[2] = h;
    }
    running += h;
  }
  __syncthreads();
}

template <bool VEC, bool BF16>
__global__ void __launch_bounds__(kFusedThreads, 1)
    mua_fused_kernel(const __grid_constant__ StepArgs A) {
  constexpr int T = kFusedThreads;
  extern __shared__ __align__(16) uint8_t dyn[];
  __shared__ FusedShared S;
  const int tid = threadIdx.x;
  const Geometry& G = A.g;
  const int j = (int)blockIdx.x;
  int64_t start;
  int L;
  block_span(A, j, start, L);
  const int k = block_k(G, L);
  uint32_t* const status = &A.hdr[kHdrStatus];

  load_weights(A, S.w1, S.w2);
  {
    const float delta = 0.0f - __uint_as_float(A.hdr[A.pair_cur]);
    const float Delta = __uint_as_float(A.hdr[A.pair_cur + 1]);
    fill_levels(S.levels, delta, __fdiv_rn(__fsub_rn(Delta, delta), 15.0f));
  }
  uint4 gv[kChunks];
  uint32_t cv[kChunks];
  load_block<T, VEC>(A.grads, A.codes, start, L, tid, gv, cv);
  __syncthreads();

  // (1) a_t, element (c, tid, e) in ab[8 c + e]; +0 past L.
  uint32_t ab[kElemsPerThread];
#pragma unroll
  for (int c = 0; c < kChunks; ++c) {
#pragma unroll
    for (int e = 0; e < kChunk; ++e) {
      const float a =
          __fadd_rn(__uint_as_float(grad_bits(gv[c], e)), S.levels[(cv[c] >> (4 * e)) & 0xFu]);
      ab[c * kChunk + e] = (elem_index<T>(c, tid, e) < L) ? __float_as_uint(a) : 0u;
    }
  }
  auto valid = [&](int c, int e) { return elem_index<T>(c, tid, e) < L; };

  // (2) exact radix select of the k-th largest key |a| over the block.
  uint32_t* hist = reinterpret_cast<uint32_t*>(dyn);  // 2048 counts
  uint32_t prefix = 0u, pmask = 0u, thr = 0u;
  int krem = k, mode = 1;
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int width = pass == 0 ? 11 : 10;
    const int shift = pass == 0 ? 20 : (pass == 1 ? 10 : 0);
    const int nbins = 1 << width;
    for (int b = tid; b < nbins; b += T) hist[b] = 0u;
    __syncthreads();
#pragma unroll
    for (int c = 0; c < kChunks; ++c) {
#pragma unroll
      for (int e = 0; e < kChunk; ++e) {
        const uint32_t key = ab[c * kChunk + e] & 0x7FFFFFFFu;
        if (valid(c, e) && (key & pmask) == prefix)
          atomicAdd(&hist[(key >> shift) & (nbins - 1)], 1u);
      }
    }
    __syncthreads();
    find_bin<T>(hist, nbins, krem, S);
    const uint32_t bin = S.res[0], above = S.res[1], inbin = S.res[2];
    prefix |= bin << shift;
    pmask |= (uint32_t)(nbins - 1) << shift;
    krem -= (int)above;
    thr = prefix;
    __syncthreads();  // S.res and hist are rewritten by the next pass
    if (inbin == (uint32_t)krem) {  // the whole bin is selected
      mode = 0;
      break;
    }
  }
  const int need = mode == 0 ? k : krem;  // mode 1: ties at thr, lowest indices first

  // Placement in index order ((c, tid, e) lexicographic): per chunk, a block
  // scan of (keys above thr, keys equal to thr) packed in 16-bit halves.
  uint32_t* row = A.window + ((int64_t)j * G.m + A.row) * G.kp;
  uint32_t selm = 0u;  // bit 8 c + e: element selected
  uint32_t run_g = 0u, run_e = 0u;
  float rmin = 0.0f, rmax = 0.0f;  // residual; selected entries become +0
  uint32_t kmax = 0u;
#pragma unroll
  for (int c = 0; c < kChunks; ++c) {
    uint32_t cg = 0u, ce = 0u;
#pragma unroll
    for (int e = 0; e < kChunk; ++e) {
      const uint32_t key = ab[c * kChunk + e] & 0x7FFFFFFFu;
      if (!valid(c, e)) continue;
      kmax = max(kmax, key);
      if (mode == 0) {
        cg += key >= thr;
      } else {
        cg += key > thr;
        ce += key == thr;
      }
    }
    const uint32_t packed = cg | (ce << 16);
    uint32_t total;
    const uint32_t incl = block_scan_1bar<T, uint32_t>(packed, S.scan, total);
    uint32_t g = run_g + ((incl - packed) & 0xFFFFu);
    uint32_t q = run_e + ((incl - packed) >> 16);
#pragma unroll
    for (int e = 0; e < kChunk; ++e) {
      const uint32_t bits = ab[c * kChunk + e];
      const uint32_t key = bits & 0x7FFFFFFFu;
      if (!valid(c, e)) continue;
      const uint32_t idx = (uint32_t)elem_index<T>(c, tid, e);
      const bool gt = (mode == 0) ? key >= thr : key > thr;
      bool sel = false;
      uint32_t pos = 0u;
      if (gt) {
        pos = g + min(q, (uint32_t)need);
        ++g;
        sel = true;
      } else if (mode == 1 && key == thr) {
        if (q < (uint32_t)need) {
          pos = g + q;
          sel = true;
        }
        ++q;
      }
      if (sel) {
        if (pos < (uint32_t)k) {
          const uint32_t vb = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(bits)));
          row[pos] = (idx & 0xFFFFu) | (vb << 16);
        }
        selm |= 1u << (c * kChunk + e);
      } else {
        rmin = fminf(rmin, __uint_as_float(bits));
        rmax = fmaxf(rmax, __uint_as_float(bits));
      }
    }
    run_g += total & 0xFFFFu;
    run_e += total >> 16;
    __syncthreads();  // S.scan is reused by the next chunk's scan
  }
  for (int sl = k + tid; sl < G.kp; sl += T) row[sl] = kEmptySlot;
  __syncthreads();  // the histogram is done with; the new row is written
  update_prefetch_rows<T>(A, j, dyn);  // the window rows land during the barrier

  // (3) block min/max and the non-finite check, one atomic pair per CTA.
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    rmin = fminf(rmin, __shfl_xor_sync(0xFFFFFFFFu, rmin, o));
    rmax = fmaxf(rmax, __shfl_xor_sync(0xFFFFFFFFu, rmax, o));
    kmax = max(kmax, __shfl_xor_sync(0xFFFFFFFFu, kmax, o));
  }
  if ((tid & 31) == 0) {
    S.mn[tid >> 5] = rmin;
    S.mx[tid >> 5] = rmax;
    S.km[tid >> 5] = kmax;
  }
  __syncthreads();
  if (tid == 0) {
    float bmin = S.mn[0], bmax = S.mx[0];
    uint32_t km = S.km[0];
    for (int w = 1; w < T / 32; ++w) {
      bmin = fminf(bmin, S.mn[w]);
      bmax = fmaxf(bmax, S.mx[w]);
      km = max(km, S.km[w]);
    }
    if (km >= kKeyInf) atomicOr(status, kStatusNonFinite);
    atomicMax(&A.hdr[A.pair_next], __float_as_uint(0.0f - bmin));  // >= +0, canonical zero
    atomicMax(&A.hdr[A.pair_next + 1], __float_as_uint(bmax + 0.0f));
    // (4) grid barrier, bounded by the global timer.
    __threadfence();
    atomicAdd(&A.hdr[kHdrBarrier], 1u);
    const uint64_t t0 = global_ns();
    uint32_t ok = 1u;
    while (ld_acquire_u32(&A.hdr[kHdrBarrier]) < (uint32_t)G.nb) {
      if (A.wait_ns == 0 || global_ns() - t0 > A.wait_ns) {  // limit 0: give up at once
        ok = 0u;
        break;
      }
      __nanosleep(100);
    }
    if (!ok) atomicOr(status, kStatusTimeout);
    __threadfence();
    S.go = ok;
  }
  __syncthreads();
  if (!S.go) return;

  // (5) e_{t+1} = Q(residual, delta_{t+1}, Delta_{t+1}) from the registers.
  const float dn = 0.0f - __uint_as_float(__ldcg(&A.hdr[A.pair_next]));
  const float Dn = __uint_as_float(__ldcg(&A.hdr[A.pair_next + 1]));
  const float inv16 =
      (Dn == dn) ? 0.0f : __fmul_rn(__fdiv_rn(15.0f, __fsub_rn(Dn, dn)), 65536.0f);
  const uint64_t dn2 = f2_pack(dn, dn), inv2 = f2_pack(inv16, inv16);
  const uint32_t big0 = quantize_big_zero(dn, inv16);
#pragma unroll
  for (int c = 0; c < kChunks; ++c) {
    const int e0 = elem_index<T>(c, tid, 0);
    if (e0 >= L) continue;
    const uint32_t selbits = (selm >> (c * kChunk)) & 0xFFu;
    uint32_t pack = 0u;
    uint8_t* cdst = A.codes + ((start + e0) >> 1);
    if (VEC) {
      const uint64_t grp = (uint64_t)(G.base_index + start + e0) >> 3;
      const uint4 x = philox4x32_10((uint32_t)grp, (uint32_t)(grp >> 32), A.t_lo, A.t_hi, A.keys);
      uint64_t a2[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        a2[i] = ((uint64_t)ab[c * kChunk + 2 * i + 1] << 32) | ab[c * kChunk + 2 * i];
      pack = quantize8(a2, selbits, x, dn2, inv2, big0);
    } else {
      const int64_t gidx = G.base_index + start + e0;
#pragma unroll
      for (int e = 0; e < kChunk; ++e) {
        float a = __uint_as_float(ab[c * kChunk + e]);
        if ((selbits >> e) & 1u) a = 0.0f;
        const float s16 = __fmul_rn(__fsub_rn(a, dn), inv16);
        const uint64_t gi = (uint64_t)gidx + e;
        const uint64_t grp = gi >> 3;
        const uint4 x = philox4x32_10((uint32_t)grp, (uint32_t)(grp >> 32), A.t_lo, A.t_hi, A.keys);
        const uint32_t xw = chunk_word(x, (int)((gi >> 1) & 3));
        const uint32_t r = (gi & 1) ? (xw >> 16) : (xw & 0xFFFFu);
        pack |= ((quantize_code_hi(s16, r) >> 16) & 0xFu) << (4 * e);
      }
    }
    if (VEC && e0 + kChunk <= L) {
      *reinterpret_cast<uint32_t*>(cdst) = pack;
    } else {
      const int nval = min(kChunk, L - e0);  // nibbles past the block's end stay 0
      if (nval < kChunk) pack &= (1u << (4 * nval)) - 1u;
      for (int e = 0; e < nval; e += 2) cdst[e >> 1] = (uint8_t)(pack >> (4 * e));
    }
  }

  // (6) AdamStats update of the block (reads the row written above).
  __syncthreads();
  block_update<T, BF16>(A, j, start, L, dyn, S.w1, S.w2);
}

}  // namespace

uint32_t fused_smem_bytes(int Bd, int kp, int m) {
  const uint32_t hist = 4u * 2048u;
  const uint32_t upd = update_smem_bytes(kFusedThreads, Bd, kp, m);
  return hist > upd ? hist : upd;
}

using FusedKernel = void (*)(const StepArgs);

FusedKernel fused_kernel(bool vec, bool bf16) {
  return bf16 ? (vec ? mua_fused_kernel<true, true> : mua_fused_kernel<false, true>)
              : (vec ? mua_fused_kernel<true, false> : mua_fused_kernel<false, false>);
}

uint32_t fused_opted[4][kMaxDevices] = {};  // per kernel instance and device

int fused_max_blocks(int Bd, int kp, int m, bool vec, bool bf16) {
  if (Bd > kFusedElems) return 0;
  const uint32_t smem = fused_smem_bytes(Bd, kp, m);
  const FusedKernel kern = fused_kernel(vec, bf16);
  if (opt_in_smem(kern, smem, fused_opted[(bf16 ? 2 : 0) + (vec ? 1 : 0)]) != cudaSuccess)
    return 0;
  int dev = 0, sms = 0, per_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kFusedThreads, smem) !=
      cudaSuccess)
    return 0;
  return per_sm * sms;
}

cudaError_t launch_fused(const StepArgs& args, bool vec, cudaStream_t stream) {
  const bool bf16 = args.params16 != nullptr;
  const FusedKernel kern = fused_kernel(vec, bf16);
  const uint32_t smem = fused_smem_bytes(args.g.Bd, args.g.kp, args.g.m);
  cudaError_t e = opt_in_smem(kern, smem, fused_opted[(bf16 ? 2 : 0) + (vec ? 1 : 0)]);
  if (e != cudaSuccess) return e;
  void* kargs[] = {const_cast<StepArgs*>(&args)};
  return cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(kern), dim3(args.g.nb),
                                     dim3(kFusedThreads), kargs, smem, stream);
}

}  // namespace mua
