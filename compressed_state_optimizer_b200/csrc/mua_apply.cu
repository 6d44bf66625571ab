// Stage kernel 2 of the MicroAdam step ([MicroAdam ¶1] = paragraph 1 of
// "MicroAdam (Sparse-Gradient Adaptive Optimization with Quantized Error
// Feedback)"), one CTA per block of B_d parameters (in passes of 32 T elements), once the select kernel has
// written every block's new window row and the global (delta_{t+1},
// Delta_{t+1}) is final:
//   e_{t+1} = Q(a_t, delta_{t+1}, Delta_{t+1}): a_t is recomputed bit for bit
//     from g_t and e_t, the entries of the new row are zeroed, and every value
//     is stochastically rounded to one of 16 levels with a 16-bit Philox4x32-10
//     draw keyed on (seed; element/8, t); codes are packed and stored in place;
//   and, for the blocks the select kernel left (j & 7 >= update_split), the
//   AdamStats update of the block's parameters (block_update).
// Blocks run in reverse order, so the first blocks find the tail of the
// select kernel's reads in L2. HBM traffic per parameter: 2.5 B read
// (g, e) + 0.5 B written (e); plus block_update's traffic for its blocks.
#include "mua_kernels.cuh"

namespace mua {
namespace {

// 256-thread CTAs (B_d = 16384) run 5 per SM: 48 registers, a few bytes of
// spill, measured 2.5 % faster than 4 per SM (6 per SM was slower again).
template <int T, bool VEC>
__global__ void __launch_bounds__(T, (T == 256 ? 5 : (T <= 512 ? 1024 / T : 1)))
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

  load_weights(A, s_w1, s_w2);

  uint32_t* sel = reinterpret_cast<uint32_t*>(dyn);  // [Wn] bits of the new row
  const int Wn = (G.Bd + 31) >> 5;

  // Issue the streaming loads first; they land while the new row is read.
  uint4 gv[kChunks];
  uint32_t cv[kChunks];
  load_block<T, VEC>(A.grads, A.codes, start, L, tid, gv, cv);

  const float delta = 0.0f - __uint_as_float(A.hdr[A.pair_cur]);
  const float Delta = __uint_as_float(A.hdr[A.pair_cur + 1]);
  fill_levels(s_lv, delta, __fdiv_rn(__fsub_rn(Delta, delta), 15.0f));
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
  // The block in passes of kChunks * 8 * T elements (the first pass's loads
  // were issued above).
  constexpr int kPass = kChunks * kChunk * T;
  for (int base = 0; base < L; base += kPass) {
  const int Lp = L - base;  // elements from this pass's start to the block's end
  if (base > 0) load_block<T, VEC>(A.grads, A.codes, start + base, Lp, tid, gv, cv);
  const uint64_t grp0 = (uint64_t)(G.base_index + start + base) >> 3;  // VEC: multiple of 8
#pragma unroll
  for (int c = 0; c < kChunks; ++c) {
    const int e0 = elem_index<T>(c, tid, 0);
    if (e0 >= Lp) continue;
    const int eb = base + e0;  // block-relative index of the chunk's first element
    const uint32_t selbits = (sel[eb >> 5] >> (eb & 31)) & 0xFFu;
    uint32_t pack = 0u;
    if (VEC) {
      const uint64_t grp = grp0 + (uint64_t)(c * T + tid);
      const uint4 x = philox4x32_10((uint32_t)grp, (uint32_t)(grp >> 32), A.t_lo, A.t_hi, A.keys);
      const uint64_t dn2 = f2_pack(dn, dn), inv2 = f2_pack(inv16, inv16);
      const uint64_t magic2 = f2_pack(8388608.0f, 8388608.0f);
#pragma unroll
      for (int e = 0; e < kChunk; e += 2) {  // elements e, e + 1: gradient word e / 2
        const uint32_t w = chunk_word(gv[c], e >> 1);
        const uint32_t off0 = (e == 0) ? ((cv[c] << 2) & 0x3Cu) : ((cv[c] >> (4 * e - 2)) & 0x3Cu);
        const uint32_t off1 = (cv[c] >> (4 * e + 2)) & 0x3Cu;
        const uint64_t g2 = ((uint64_t)(w & 0xFFFF0000u) << 32) | (uint32_t)(w << 16);
        const uint64_t l2 = f2_pack(*reinterpret_cast<const float*>(lvb + off0),
                                    *reinterpret_cast<const float*>(lvb + off1));
        uint64_t a2 = f2_add_rn(g2, l2);
        if ((selbits >> e) & 1u) a2 &= 0xFFFFFFFF00000000ull;  // selected: a = +0
        if ((selbits >> (e + 1)) & 1u) a2 &= 0x00000000FFFFFFFFull;
        const uint64_t big2 = f2_add_rz(f2_mul_rn(f2_sub_rn(a2, dn2), inv2), magic2);
        const uint32_t xw = chunk_word(x, e >> 1);
        // floor(s16) sits in the low mantissa of 2^23 + s16 (rounded toward zero)
        const uint32_t hi0 = __viaddmin_u32((uint32_t)big2, xw & 0xFFFFu, 0x4B0FFFFFu);
        const uint32_t hi1 = __viaddmin_u32((uint32_t)(big2 >> 32), xw >> 16, 0x4B0FFFFFu);
        pack |= (e <= 4 ? (hi0 >> (16 - 4 * e)) : (hi0 << (4 * e - 16))) & (0xFu << (4 * e));
        pack |= (e + 1 <= 4 ? (hi1 >> (12 - 4 * e)) : (hi1 << (4 * e - 12))) & (0xFu << (4 * e + 4));
      }
    } else {
      const int64_t gidx = G.base_index + start + eb;
      const uint64_t ga = (uint64_t)gidx >> 3;
      const uint4 xa = philox4x32_10((uint32_t)ga, (uint32_t)(ga >> 32), A.t_lo, A.t_hi, A.keys);
      const uint4 xb =
          philox4x32_10((uint32_t)(ga + 1), (uint32_t)((ga + 1) >> 32), A.t_lo, A.t_hi, A.keys);
#pragma unroll
      for (int e = 0; e < kChunk; ++e) {
        const float gf = __uint_as_float(grad_bits(gv[c], e));
        float a = __fadd_rn(gf, s_lv[(cv[c] >> (4 * e)) & 0xFu]);
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
    if (VEC && e0 + kChunk <= Lp) {
      *reinterpret_cast<uint32_t*>(cdst) = pack;
    } else {
      const int nval = min(kChunk, Lp - e0);  // nibbles past the block's end stay 0
      if (nval < kChunk) pack &= (1u << (4 * nval)) - 1u;
      for (int e = 0; e < nval; e += 2) cdst[e >> 1] = (uint8_t)(pack >> (4 * e));
    }
  }
  }
  if (!update_in_select(A, j)) {  // (6) AdamStats update of block j
    __syncthreads();
    block_update<T>(A, j, start, L, dyn, s_w1, s_w2);
  }
}

template <int T>
cudaError_t launch_t(const StepArgs& args, bool vec, uint32_t smem, cudaStream_t stream) {
  auto kern = vec ? mua_apply_kernel<T, true> : mua_apply_kernel<T, false>;
  if (smem > 32 * 1024) {  // opt in well below 48 KB: static arrays count too
    const cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
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
