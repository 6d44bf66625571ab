// Stage kernel 2 of the MicroAdam step ([MicroAdam ¶1] = paragraph 1 of
// "MicroAdam (Sparse-Gradient Adaptive Optimization with Quantized Error
// Feedback)"), one CTA per block of B_d parameters (in passes of 32 T
// elements), once the select kernel has written every block's new window row
// and the global (delta_{t+1}, Delta_{t+1}) is final:
//   e_{t+1} = Q(a_t, delta_{t+1}, Delta_{t+1}): a_t is recomputed bit for bit
//     from g_t and e_t, the entries of the new row are zeroed, and every value
//     is stochastically rounded to one of 16 levels with a 16-bit Philox4x32-10
//     draw keyed on (seed; element/8, t); codes are packed and stored in place;
//   then the AdamStats update of the block's parameters (block_update).
// Blocks run in reverse order, so the first blocks find the tail of the
// select kernel's reads in L2. HBM traffic per parameter: 2.5 B read
// (g, e) + 0.5 B written (e); plus block_update's traffic: the block's window
// rows and a read-modify-write of the parameters on the rows' index union.
#include "mua_kernels.cuh"

namespace mua {
namespace {

// Stage (4) for one pass of kChunks * 8 * T elements starting at block offset
// `base` (gv / cv already loaded). FULL: every element of the pass lies inside
// the block (no bounds checks); VEC: 16-byte loads and one Philox call per
// chunk of 8 (the chunk starts on a multiple of 8).
template <int T, bool VEC, bool FULL>
__device__ __forceinline__ void codec_pass(const StepArgs& A, int64_t start, int base, int L,
                                           const uint32_t* sel, const char* lvb, float dn,
                                           float inv16, uint32_t big0,
                                           const uint4 (&gv)[kChunks],
                                           const uint32_t (&cv)[kChunks]) {
  const int tid = threadIdx.x;
  const Geometry& G = A.g;
  const int Lp = L - base;  // elements from this pass's start to the block's end
  const uint64_t grp0 = (uint64_t)(G.base_index + start + base) >> 3;  // VEC: multiple of 8
#pragma unroll
  for (int c = 0; c < kChunks; ++c) {
    const int e0 = elem_index<T>(c, tid, 0);
    if (!FULL && e0 >= Lp) continue;
    const int eb = base + e0;  // block-relative index of the chunk's first element
    const uint32_t selbits = (sel[eb >> 5] >> (eb & 31)) & 0xFFu;
    uint32_t pack = 0u;
    if (VEC) {
      const uint64_t grp = grp0 + (uint64_t)(c * T + tid);
      const uint4 x = philox4x32_10((uint32_t)grp, (uint32_t)(grp >> 32), A.t_lo, A.t_hi, A.keys);
      uint64_t a2[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {  // elements 2i, 2i + 1: gradient word i, code byte i
        const uint32_t w = chunk_word(gv[c], i);
        const uint32_t b = (cv[c] >> (8 * i)) & 0xFFu;
        const uint64_t g2 = ((uint64_t)(w & 0xFFFF0000u) << 32) | (uint32_t)(w << 16);
        const uint64_t l2 =
            ((uint64_t)__float_as_uint(*reinterpret_cast<const float*>(lvb + 4 * (b >> 4))) << 32) |
            __float_as_uint(*reinterpret_cast<const float*>(lvb + 4 * (b & 15u)));
        a2[i] = f2_add_rn(g2, l2);
      }
      pack = quantize8(a2, selbits, x, f2_pack(dn, dn), f2_pack(inv16, inv16), big0);
    } else {
      const int64_t gidx = G.base_index + start + eb;
      const uint64_t ga = (uint64_t)gidx >> 3;
      const uint4 xa = philox4x32_10((uint32_t)ga, (uint32_t)(ga >> 32), A.t_lo, A.t_hi, A.keys);
      const uint4 xb =
          philox4x32_10((uint32_t)(ga + 1), (uint32_t)((ga + 1) >> 32), A.t_lo, A.t_hi, A.keys);
#pragma unroll
      for (int e = 0; e < kChunk; ++e) {
        const float gf = __uint_as_float(grad_bits(gv[c], e));
        float a = __fadd_rn(gf, *reinterpret_cast<const float*>(lvb + 4 * ((cv[c] >> (4 * e)) & 0xFu)));
        if ((selbits >> e) & 1u) a = 0.0f;
        const float s16 = __fmul_rn(__fsub_rn(a, dn), inv16);
        const uint64_t gi = (uint64_t)gidx + e;
        const uint4& x = ((gi >> 3) == ga) ? xa : xb;
        const uint32_t xw = chunk_word(x, (int)((gi >> 1) & 3));
        const uint32_t r = (gi & 1) ? (xw >> 16) : (xw & 0xFFFFu);
        const uint32_t hi = quantize_code_hi(s16, r);
        pack |= ((hi >> 16) & 0xFu) << (4 * e);
      }
    }
    uint8_t* cdst = A.codes + ((start + eb) >> 1);
    if (VEC && (FULL || e0 + kChunk <= Lp)) {
      *reinterpret_cast<uint32_t*>(cdst) = pack;
    } else {
      const int nval = min(kChunk, Lp - e0);  // nibbles past the block's end stay 0
      if (nval < kChunk) pack &= (1u << (4 * nval)) - 1u;
      for (int e = 0; e < nval; e += 2) cdst[e >> 1] = (uint8_t)(pack >> (4 * e));
    }
  }
}

// 256-thread CTAs (B_d = 16384) run 5 per SM by default: 48 registers.
#ifndef MUA_APPLY_CTAS_256
#define MUA_APPLY_CTAS_256 5
#endif
template <int T, bool VEC, bool BF16>
__global__ void __launch_bounds__(T, (T == 256 ? MUA_APPLY_CTAS_256 : (T <= 512 ? 1024 / T : 1)))
    mua_apply_kernel(const __grid_constant__ StepArgs A) {
  extern __shared__ __align__(16) uint8_t dyn[];
  __shared__ float s_lv[16];
  __shared__ float s_w1[kMaxWindow], s_w2[kMaxWindow];

  const int tid = threadIdx.x;
  const Geometry& G = A.g;
  const int j = G.nb - 1 - (int)blockIdx.x;
  int64_t start;
  int L;
  block_span(A, j, start, L);
  constexpr int kPass = kChunks * kChunk * T;
  // Every pass of a whole block lies inside it (B_d a multiple of the pass).
  const bool full = VEC && (L % kPass) == 0;

  // The block's window rows start copying into shared memory now; they land
  // while the codec runs (block_update waits for them).
  update_prefetch_rows<T>(A, j, dyn);
  load_weights(A, s_w1, s_w2);

  uint32_t* sel = reinterpret_cast<uint32_t*>(dyn);  // [Wn] bits of the new row
  const int Wn = (G.Bd + 31) >> 5;

  // Issue the streaming loads first; they land while the new row is read.
  uint4 gv[kChunks];
  uint32_t cv[kChunks];
  if (full) load_block<T, VEC, true>(A.grads, A.codes, start, L, tid, gv, cv);
  else load_block<T, VEC>(A.grads, A.codes, start, L, tid, gv, cv);

  const float delta = 0.0f - __uint_as_float(A.hdr[A.pair_cur]);
  const float Delta = __uint_as_float(A.hdr[A.pair_cur + 1]);
  const float unit = __fdiv_rn(__fsub_rn(Delta, delta), 15.0f);
  fill_levels(s_lv, delta, unit);
  for (int w = tid; w < Wn; w += T) sel[w] = 0u;
  __syncthreads();
  {
    const uint32_t* row = A.window + ((int64_t)j * G.m + A.row) * G.kp;
    for (int s = tid; s < G.kp; s += T) {
      const uint32_t idx = row[s] & 0xFFFFu;
      if (idx < (uint32_t)L) atomicOr(&sel[idx >> 5], 1u << (idx & 31));  // 0xFFFF: empty
    }
  }
  __syncthreads();

  // e_{t+1} = Q(a_t with the new row zeroed, delta_{t+1}, Delta_{t+1}).
  const float dn = 0.0f - __uint_as_float(A.hdr[A.pair_next]);
  const float Dn = __uint_as_float(A.hdr[A.pair_next + 1]);
  const float inv16 =
      (Dn == dn) ? 0.0f : __fmul_rn(__fdiv_rn(15.0f, __fsub_rn(Dn, dn)), 65536.0f);
  const char* lvb = reinterpret_cast<const char*>(s_lv);
  const uint32_t big0 = quantize_big_zero(dn, inv16);
  // The block in passes of kPass elements (the first pass's loads were issued
  // above).
  if (full) {
    for (int base = 0; base < L; base += kPass) {
      if (base > 0) load_block<T, VEC, true>(A.grads, A.codes, start + base, L - base, tid, gv, cv);
      codec_pass<T, VEC, true>(A, start, base, L, sel, lvb, dn, inv16, big0, gv, cv);
    }
  } else {
    for (int base = 0; base < L; base += kPass) {
      if (base > 0) load_block<T, VEC>(A.grads, A.codes, start + base, L - base, tid, gv, cv);
      codec_pass<T, VEC, false>(A, start, base, L, sel, lvb, dn, inv16, big0, gv, cv);
    }
  }
  __syncthreads();  // (6) AdamStats update of block j
  block_update<T, BF16>(A, j, start, L, dyn, s_w1, s_w2);
}

template <int T>
cudaError_t launch_t(const StepArgs& args, bool vec, uint32_t smem, cudaStream_t stream) {
  const bool bf16 = args.params16 != nullptr;
  auto kern = bf16 ? (vec ? mua_apply_kernel<T, true, true> : mua_apply_kernel<T, false, true>)
                   : (vec ? mua_apply_kernel<T, true, false> : mua_apply_kernel<T, false, false>);
  static uint32_t opted[4][kMaxDevices] = {};
  const cudaError_t e = opt_in_smem(kern, smem, opted[(bf16 ? 2 : 0) + (vec ? 1 : 0)]);
  if (e != cudaSuccess) return e;
  kern<<<args.g.nb, T, smem, stream>>>(args);
  return cudaGetLastError();
}

}  // namespace

uint32_t apply_smem_bytes(int threads, int Bd, int kp, int m) {
  const uint32_t own = 4u * (uint32_t)((Bd + 31) / 32);
  const uint32_t upd = update_smem_bytes(threads, Bd, kp, m);
  return own > upd ? own : upd;
}

cudaError_t launch_apply(const StepArgs& args, int threads, bool vec, uint32_t smem,
                         cudaStream_t stream) {
  switch (threads) {
    case 32: return launch_t<32>(args, vec, smem, stream);
    case 64: return launch_t<64>(args, vec, smem, stream);
    case 128: return launch_t<128>(args, vec, smem, stream);
    case 256: return launch_t<256>(args, vec, smem, stream);
    case 512: return launch_t<512>(args, vec, smem, stream);
    case 1024: return launch_t<1024>(args, vec, smem, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace mua
