// Stage kernel 2 of the MicroAdam step ([MicroAdam ¶1] = paragraph 1 of
// "MicroAdam (Sparse-Gradient Adaptive Optimization with Quantized Error
// Feedback)"), one CTA per block of B_d parameters, after the select kernel
// has written the block's new window row and the global (delta_{t+1},
// Delta_{t+1}) is final:
//   e_{t+1} = Q(a_t, delta_{t+1}, Delta_{t+1}): a_t is recomputed bit for bit
//     from g_t and e_t, the entries of the new row are zeroed, and every value
//     is stochastically rounded to one of 16 levels with a Philox4x32-10 draw
//     keyed on (seed; element/8, t); codes are packed in place;
//   m_hat = AdamStats(beta1, G), v_hat = AdamStats(beta2, G^2): the block's
//     window entries are staged in shared memory, their index union is ranked
//     with a bitmask + popcount prefix, and the entries of each index are
//     linked into a per-index list, summed oldest row first (deterministic);
//   p <- p*(1 - lr*wd) (dense, only when wd != 0), then
//   p <- p - lr * m_hat / (eps + sqrt(v_hat)) on the union.
// HBM traffic per parameter: 2.5 B read (g, e) + 0.5 B written (e); per window
// entry 4 B read; per union index one fp32 read-modify-write of the parameter.
#include "mua_kernels.cuh"

namespace mua {
namespace {

constexpr uint32_t kNil = 0xFFFFFFFFu;

struct ApplySmem {
  uint32_t* mask;  // [Wn]  bit i: index i is in the window's union
  uint32_t* sel;   // [Wn]  bit i: index i is in the new row (zeroed in e_{t+1})
  uint32_t* wpre;  // [Wn]  popcount prefix of mask
  uint32_t* W;     // [E]   staged window entries, age-major: e = age*kp + slot
  uint32_t* nxt;   // [E]   list links: (age << 16) | entry, kNil ends a list
  uint32_t* head;  // [Ucap] list heads per union rank
  uint32_t* scan;  // [T/32]
};

__device__ __forceinline__ ApplySmem carve(uint8_t* base, int Wn, int E, int Ucap, int nw) {
  ApplySmem s;
  uint32_t* p = reinterpret_cast<uint32_t*>(base);
  s.mask = p; p += Wn;
  s.sel = p; p += Wn;
  s.wpre = p; p += Wn;
  s.W = p; p += E;
  s.nxt = p; p += E;
  s.head = p; p += Ucap;
  s.scan = p; p += nw;
  return s;
}

template <int T, bool VEC>
__global__ void __launch_bounds__(T) mua_apply_kernel(const ApplyArgs A) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const int tid = threadIdx.x;
  const Geometry& G = A.g;
  const int j = A.reverse ? (G.nb - 1 - (int)blockIdx.x) : (int)blockIdx.x;
  const int64_t start = (int64_t)j * G.Bd;
  const int L = (j == G.nb - 1) ? G.last_len : G.Bd;
  const int Wn = (G.Bd + 31) >> 5;
  const int E = G.m * G.kp;
  const int Ucap = min(G.Bd, E);
  const ApplySmem S = carve(smem_raw, Wn, E, Ucap, T / 32);
  __shared__ float s_w1[kMaxWindow], s_w2[kMaxWindow];
  if (tid == 0) {  // constant indices: the weights stay in the parameter bank
#pragma unroll
    for (int r = 0; r < kMaxWindow; ++r) {
      s_w1[r] = A.w1[r];
      s_w2[r] = A.w2[r];
    }
  }

  // Issue the streaming loads first; they land while the window is ranked.
  uint4 gv[kChunks];
  uint32_t cv[kChunks];
  load_block<T, VEC>(A.grads, A.codes, start, L, tid, gv, cv);

  for (int w = tid; w < Wn; w += T) {
    S.mask[w] = 0u;
    S.sel[w] = 0u;
  }
  for (int u = tid; u < Ucap; u += T) S.head[u] = kNil;
  __syncthreads();

  // Stage the rows of steps t, t-1, ..., t-rows+1 (age 0 = this step's row).
  const uint32_t* wblk = A.window + (int64_t)j * G.m * G.kp;
  const int staged = A.rows * G.kp;
  for (int e = tid; e < staged; e += T) {
    const int age = e / G.kp;
    const int slot = e - age * G.kp;
    int phys = A.row - age;
    if (phys < 0) phys += G.m;
    const uint32_t v = wblk[phys * G.kp + slot];
    S.W[e] = v;
    const uint32_t idx = v & 0xFFFFu;
    if (idx < (uint32_t)L) {  // 0xFFFF marks an empty slot
      atomicOr(&S.mask[idx >> 5], 1u << (idx & 31));
      if (age == 0) atomicOr(&S.sel[idx >> 5], 1u << (idx & 31));
    }
  }
  __syncthreads();

  // Rank of each union index: popcount prefix over the mask words (Wn <= T).
  const uint32_t pc = (tid < Wn) ? (uint32_t)__popc(S.mask[tid]) : 0u;
  uint32_t U;
  const uint32_t incl = block_inclusive_scan<T, uint32_t>(pc, S.scan, U);
  if (tid < Wn) S.wpre[tid] = incl - pc;
  __syncthreads();

  // Link every window entry into the list of its union rank.
  for (int e = tid; e < staged; e += T) {
    const uint32_t idx = S.W[e] & 0xFFFFu;
    if (idx >= (uint32_t)L) continue;
    const uint32_t w = idx >> 5;
    const uint32_t rank = S.wpre[w] + (uint32_t)__popc(S.mask[w] & ((1u << (idx & 31)) - 1u));
    const uint32_t age = (uint32_t)(e / G.kp);
    S.nxt[e] = atomicExch(&S.head[rank], (age << 16) | (uint32_t)e);
  }

  // e_{t+1} = Q(a_t with the new row zeroed, delta_{t+1}, Delta_{t+1}).
  {
    const float delta = 0.0f - __uint_as_float(A.hdr[A.pair_cur]);
    const float Delta = __uint_as_float(A.hdr[A.pair_cur + 1]);
    const float unit = __fdiv_rn(__fsub_rn(Delta, delta), 15.0f);
    const float dn = 0.0f - __uint_as_float(A.hdr[A.pair_next]);
    const float Dn = __uint_as_float(A.hdr[A.pair_next + 1]);
    const float inv = (Dn == dn) ? 0.0f : __fdiv_rn(15.0f, __fsub_rn(Dn, dn));
#pragma unroll
    for (int c = 0; c < kChunks; ++c) {
      const int e0 = elem_index<T>(c, tid, 0);
      if (e0 >= L) continue;
      const uint32_t selbits = (S.sel[e0 >> 5] >> (e0 & 31)) & 0xFFu;
      const int64_t gidx = G.base_index + start + e0;
      uint4 xa, xb;
      if (VEC) {
        const uint64_t grp = (uint64_t)gidx >> 3;
        xa = philox4x32_10((uint32_t)grp, (uint32_t)(grp >> 32), A.t_lo, A.t_hi, A.keys);
        xb = xa;
      } else {
        const uint64_t ga = (uint64_t)gidx >> 3, gb = (uint64_t)(gidx + 7) >> 3;
        xa = philox4x32_10((uint32_t)ga, (uint32_t)(ga >> 32), A.t_lo, A.t_hi, A.keys);
        xb = philox4x32_10((uint32_t)gb, (uint32_t)(gb >> 32), A.t_lo, A.t_hi, A.keys);
      }
      const uint64_t ga8 = (uint64_t)gidx >> 3;
      uint32_t pack = 0u;
#pragma unroll
      for (int e = 0; e < kChunk; ++e) {
        const uint32_t word = chunk_word(gv[c], e >> 1);
        const uint32_t gb = (e & 1) ? (word >> 16) : (word & 0xFFFFu);
        const uint32_t code = (cv[c] >> (4 * e)) & 0xFu;
        float a = dequant_add(gb, code, delta, unit);
        if ((selbits >> e) & 1u) a = 0.0f;
        const float s = __fmul_rn(__fsub_rn(a, dn), inv);
        const uint64_t gi = (uint64_t)gidx + e;
        const uint4& x = ((gi >> 3) == ga8) ? xa : xb;
        const uint32_t xw = chunk_word(x, (int)((gi >> 1) & 3));
        const uint32_t r16 = (gi & 1) ? (xw >> 16) : (xw & 0xFFFFu);
        const float xi = __fmul_rn(__uint2float_rn(r16), 1.0f / 65536.0f);
        const float y = __fadd_rn(s, xi);
        uint32_t q = 0u;
        if (y >= 1.0f) q = (uint32_t)min(15, __float2int_rd(y));
        pack |= q << (4 * e);
      }
      uint8_t* cdst = A.codes + ((start + e0) >> 1);
      if (VEC && e0 + kChunk <= L) {
        *reinterpret_cast<uint32_t*>(cdst) = pack;
      } else {
        for (int e = 0; e < kChunk && e0 + e < L; e += 2) cdst[e >> 1] = (uint8_t)(pack >> (4 * e));
      }
      if (A.has_decay) {
        float* pd = A.params + start + e0;
        for (int e = 0; e < kChunk && e0 + e < L; ++e) pd[e] = __fmul_rn(pd[e], A.decay);
      }
    }
  }
  __syncthreads();

  // AdamStats per union index, oldest row first, then the update.
  for (uint32_t r = tid; r < U; r += T) {
    const uint32_t head = S.head[r];
    float z1 = 0.0f, z2 = 0.0f;
    uint32_t idx = 0u;
    int prev = 1 << 30;
    for (;;) {
      int best = -1;
      uint32_t bv = 0u;
      for (uint32_t l = head; l != kNil; l = S.nxt[l & 0xFFFFu]) {
        const int age = (int)(l >> 16);
        if (age < prev && age > best) {
          best = age;
          bv = S.W[l & 0xFFFFu];
        }
      }
      if (best < 0) break;
      const float V = __uint_as_float(bv & 0xFFFF0000u);
      z1 = __fadd_rn(z1, __fmul_rn(s_w1[best], V));
      z2 = __fadd_rn(z2, __fmul_rn(s_w2[best], __fmul_rn(V, V)));
      idx = bv & 0xFFFFu;
      prev = best;
    }
    const float mh = __fmul_rn(A.f1, z1);
    const float vh = __fmul_rn(A.f2, z2);
    const float u = __fdiv_rn(mh, __fadd_rn(A.eps, __fsqrt_rn(vh)));
    float* pp = A.params + start + idx;
    *pp = __fsub_rn(*pp, __fmul_rn(A.lr, u));
    if (A.mhat) A.mhat[start + idx] = mh;
    if (A.vhat) A.vhat[start + idx] = vh;
  }
}

template <int T>
cudaError_t launch_t(const ApplyArgs& args, bool vec, cudaStream_t stream) {
  auto kern = vec ? mua_apply_kernel<T, true> : mua_apply_kernel<T, false>;
  if (args.smem_bytes > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(
        kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)args.smem_bytes);
    if (e != cudaSuccess) return e;
  }
  kern<<<args.g.nb, T, args.smem_bytes, stream>>>(args);
  return cudaGetLastError();
}

}  // namespace

uint32_t apply_smem_bytes(int threads, int Bd, int kp, int m) {
  const int Wn = (Bd + 31) / 32;
  const int E = m * kp;
  const int Ucap = Bd < E ? Bd : E;
  return (uint32_t)(4 * (3 * Wn + 2 * E + Ucap + threads / 32));
}

cudaError_t launch_apply(const ApplyArgs& args, int threads, bool vec, cudaStream_t stream) {
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
