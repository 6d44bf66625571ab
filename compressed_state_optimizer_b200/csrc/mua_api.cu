// Host side of libmua.so: the C ABI declared in include/mua.h.
//
// [MicroAdam ¶n] is paragraph n of "MicroAdam (Sparse-Gradient Adaptive
// Optimization with Quantized Error Feedback)".
//
// A handle holds geometry only. mua_step enqueues, on the caller's stream:
//   1. an 8-byte memset of the (-delta_{t+1}, Delta_{t+1}) accumulator pair,
//   2. the select kernel, one warp per block (mua_select_warp.cu),
//   3. the apply kernel (one CTA per block, reverse block order so the tail
//      of the select kernel's reads is still in L2): codec, then the
//      AdamStats update of the block (mua_apply.cu).
// Everything the kernels need per step (beta^r weights, bias corrections,
// Philox round keys) is computed here in fp64 and rounded once to fp32 /
// uint32 before launch.
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <new>

#include "../../include/mua.h"
#include "mua_kernels.cuh"

static_assert(mua::kMaxSegments == MUA_MAX_SEGMENTS, "segment table size");

struct mua_ctx {
  int64_t d;            // elements of this handle
  int64_t d_total;      // elements of the whole vector
  int64_t block_begin;  // first global block
  int64_t nb;           // blocks of this handle
  int32_t Bd, kb, kp, m;
  int32_t last_len;
  int32_t apply_threads; // CTA size of the apply kernel (two passes per block from B_d 2048)
  bool vec;             // 16-byte vector path usable (B_d % 8 == 0)
  int64_t off_codes, off_window, bytes;
  uint32_t apply_smem;
  bool whole;           // the handle covers the whole vector (not one shard of it)
  int64_t wait_ns;      // bound on a grid-barrier wait (fused step)
  int32_t fused_cap[2][mua::kMaxDevices];  // co-resident fused CTAs [bf16][device] (-1: unknown)
  // Tensor list cut per tensor (n_seg > 0; whole vector, not a shard).
  int32_t n_seg;
  int32_t seg_first[mua::kMaxSegments];
  int64_t seg_start[mua::kMaxSegments];
  int64_t seg_len[mua::kMaxSegments];
};

namespace {

thread_local char g_cuda_err[256] = "no CUDA error";

// Default bound on the fused step's grid-barrier wait: far above a step's
// duration, far below anything that would look like a hang.
constexpr int64_t kDefaultWaitNs = 2000000000;

int cuda_fail(cudaError_t e, const char* where) {
  std::snprintf(g_cuda_err, sizeof g_cuda_err, "%s: %s", where, cudaGetErrorString(e));
  return MUA_ERR_CUDA;
}

int64_t round_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

int pick_threads(int Bd) {
  const int need = (Bd + mua::kElemsPerThread - 1) / mua::kElemsPerThread;
  int t = 32;
  while (t < need) t <<= 1;
  return t;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Warps of the apply kernel resident per SM at CTA size T: limited by its
// launch bound (5 CTAs of 256, else 1024 / T CTAs), by shared memory (228 KB
// per SM, 1 KB reserved per CTA) and by 2048 threads.
int apply_warps_per_sm(int T, int Bd, int kp, int m) {
  const int by_bound = T == 256 ? 5 : (T <= 512 ? 1024 / T : 1);
  const int by_smem = (228 * 1024) / ((int)mua::apply_smem_bytes(T, Bd, kp, m) + 1024);
  const int by_threads = 2048 / T;
  return std::min(by_bound, std::min(by_smem, by_threads)) * (T / 32);
}

// Half of T, the CTA that holds a block in one pass (the block then takes two
// passes; more CTAs per SM, so one CTA's update barriers overlap the others'
// codec work), unless the update's shared memory makes the full CTA keep more
// warps resident (long windows).
int pick_apply_threads(int T, int Bd, int kp, int m) {
  if (T < 64) return T;
  return apply_warps_per_sm(T / 2, Bd, kp, m) >= apply_warps_per_sm(T, Bd, kp, m) ? T / 2 : T;
}

int make(int64_t d_total, int32_t Bd, int32_t kb, int32_t m, int32_t bits,
         int64_t block_begin, int64_t block_count, mua_t* out) {
  if (!out) return MUA_ERR_ARG;
  *out = nullptr;
  if (d_total < 1 || Bd < 2 || Bd > 32766 || (Bd & 1) || kb < 1 || kb > Bd || m < 1 ||
      m > mua::kMaxWindow)
    return MUA_ERR_ARG;
  if (bits != 4) return MUA_ERR_UNSUPPORTED;
  const int64_t nb_total = (d_total + Bd - 1) / Bd;
  if (block_begin < 0 || block_count < 1 || block_begin + block_count > nb_total)
    return MUA_ERR_ARG;
  if (block_count > 0x7FFFFFFF) return MUA_ERR_UNSUPPORTED;
  const int32_t kp = (int32_t)round_up(kb, 4);
  if ((int64_t)m * kp > mua::kMaxWindowEntries) return MUA_ERR_UNSUPPORTED;

  mua_ctx* h = new (std::nothrow) mua_ctx();
  if (!h) return MUA_ERR_ARG;
  h->d_total = d_total;
  h->block_begin = block_begin;
  h->nb = block_count;
  const int64_t first = block_begin * Bd;
  const int64_t last_end = std::min<int64_t>(d_total, (block_begin + block_count) * Bd);
  h->d = last_end - first;
  h->Bd = Bd;
  h->kb = kb;
  h->kp = kp;
  h->m = m;
  h->last_len = (int32_t)(h->d - (block_count - 1) * Bd);
  h->apply_threads = pick_apply_threads(pick_threads(Bd), Bd, kp, m);
  h->vec = (Bd % 8) == 0;
  h->off_codes = 256;
  h->off_window = h->off_codes + round_up((h->d + 1) / 2, 256);
  h->bytes = h->off_window + 4 * block_count * (int64_t)m * kp;
  h->apply_smem = mua::apply_smem_bytes(h->apply_threads, Bd, kp, m);
  h->whole = (block_begin == 0 && block_count == nb_total);
  h->wait_ns = kDefaultWaitNs;
  for (int i = 0; i < mua::kMaxDevices; ++i) h->fused_cap[0][i] = h->fused_cap[1][i] = -1;
  h->n_seg = 0;
  *out = h;
  return MUA_OK;
}

int make_segmented(const int64_t* seg_len, int32_t n_seg, int32_t Bd, int32_t kb, int32_t m,
                   int32_t bits, mua_t* out) {
  if (!out) return MUA_ERR_ARG;
  *out = nullptr;
  if (!seg_len || n_seg < 1) return MUA_ERR_ARG;
  if (n_seg > mua::kMaxSegments) return MUA_ERR_UNSUPPORTED;
  int64_t d = 0, nb = 0;
  bool all8 = true;
  for (int32_t s = 0; s < n_seg; ++s) {
    if (seg_len[s] < 1) return MUA_ERR_ARG;
    if (seg_len[s] & 1) return MUA_ERR_UNSUPPORTED;  // blocks must start on a code byte
    if (Bd >= 2) nb += (seg_len[s] + Bd - 1) / Bd;
    all8 = all8 && (seg_len[s] % 8) == 0;
    d += seg_len[s];
  }
  if (nb > 0x7FFFFFFF) return MUA_ERR_UNSUPPORTED;
  // The flat geometry of the same d and block count checks the other
  // arguments and sizes the state; the segment table then replaces the cut.
  mua_t h = nullptr;
  int rc = make(d, Bd, kb, m, bits, 0, (d + Bd - 1) / Bd, &h);
  if (rc != MUA_OK) return rc;
  h->nb = nb;
  h->bytes = h->off_window + 4 * nb * (int64_t)m * h->kp;
  h->vec = h->vec && all8;
  h->n_seg = n_seg;
  int64_t first = 0, start = 0;
  for (int32_t s = 0; s < n_seg; ++s) {
    h->seg_first[s] = (int32_t)first;
    h->seg_start[s] = start;
    h->seg_len[s] = seg_len[s];
    first += (seg_len[s] + Bd - 1) / Bd;
    start += seg_len[s];
  }
  const int64_t last = seg_len[n_seg - 1];
  h->last_len = (int32_t)(last - ((last + Bd - 1) / Bd - 1) * (int64_t)Bd);
  *out = h;
  return MUA_OK;
}

bool finite_f(float x) { return std::isfinite(x); }

int check_hyper(float lr, float beta1, float beta2, float eps, float wd, int64_t t) {
  if (t < 1) return MUA_ERR_ARG;
  // eps > 0: with eps = 0 an index whose window values are all zero would give
  // m_hat / sqrt(v_hat) = 0 / 0.
  if (!finite_f(lr) || !finite_f(wd) || !finite_f(eps) || !(eps > 0.0f)) return MUA_ERR_ARG;
  if (!(beta1 >= 0.0f && beta1 < 1.0f) || !(beta2 >= 0.0f && beta2 < 1.0f)) return MUA_ERR_ARG;
  return MUA_OK;
}

mua::Geometry geometry(const mua_ctx* h) {
  mua::Geometry g;
  g.d = h->d;
  g.base_index = h->block_begin * h->Bd;
  g.Bd = h->Bd;
  g.kb = h->kb;
  g.kp = h->kp;
  g.m = h->m;
  g.nb = (int32_t)h->nb;
  g.last_len = h->last_len;
  return g;
}

// Header word of the (-delta, Delta) pair holding step s's scalars.
int pair_word(int64_t s) { return (s & 1) ? mua::kHdrPair1 : mua::kHdrPair0; }

}  // namespace

extern "C" {

int mua_create(int64_t d, int32_t block_size, int32_t k_per_block, int32_t window,
               int32_t bits, mua_t* out) {
  if (d < 1 || block_size < 2) {
    if (out) *out = nullptr;
    return MUA_ERR_ARG;
  }
  return make(d, block_size, k_per_block, window, bits, 0, (d + block_size - 1) / block_size,
              out);
}

int mua_create_shard(int64_t d_total, int32_t block_size, int32_t k_per_block, int32_t window,
                     int32_t bits, int64_t block_begin, int64_t block_count, mua_t* out) {
  return make(d_total, block_size, k_per_block, window, bits, block_begin, block_count, out);
}

int mua_create_segmented(const int64_t* seg_len, int32_t n_seg, int32_t block_size,
                         int32_t k_per_block, int32_t window, int32_t bits, mua_t* out) {
  return make_segmented(seg_len, n_seg, block_size, k_per_block, window, bits, out);
}

void mua_destroy(mua_t h) { delete h; }

int64_t mua_state_bytes(mua_t h) { return h ? h->bytes : MUA_ERR_ARG; }

int mua_state_layout(mua_t h, int64_t* out) {
  if (!h || !out) return MUA_ERR_ARG;
  out[MUA_LAYOUT_HEADER] = 0;
  out[MUA_LAYOUT_CODES] = h->off_codes;
  out[MUA_LAYOUT_WINDOW] = h->off_window;
  out[MUA_LAYOUT_ROW_STRIDE] = h->kp;
  out[MUA_LAYOUT_BLOCKS] = h->nb;
  out[MUA_LAYOUT_BYTES] = h->bytes;
  return MUA_OK;
}

int64_t mua_minmax_offset(mua_t h, int64_t t) {
  if (!h || t < 1) return MUA_ERR_ARG;
  return 4 * (int64_t)pair_word(t + 1);
}

// params: fp32[d] or, with bf16, bf16[d] bits; it may be NULL only for
// mua_select (which does not touch it).
static int fill_args(mua_t h, void* params, bool bf16, const uint16_t* grads, void* state,
                     float lr, float beta1, float beta2, float eps, float wd, int64_t t,
                     uint64_t seed, float* mhat, float* vhat, mua::StepArgs* out,
                     bool params_optional = false) {
  if (!h || (!params && !params_optional) || !grads || !state) return MUA_ERR_ARG;
  const int rc = check_hyper(lr, beta1, beta2, eps, wd, t);
  if (rc != MUA_OK) return rc;
  if (!aligned16(params) || !aligned16(grads) || !aligned16(state)) return MUA_ERR_ALIGN;
  if ((mhat && !aligned16(mhat)) || (vhat && !aligned16(vhat))) return MUA_ERR_ALIGN;
  uint8_t* st = static_cast<uint8_t*>(state);
  mua::StepArgs& A = *out;
  std::memset(&A, 0, sizeof A);
  A.g = geometry(h);
  A.params = bf16 ? nullptr : static_cast<float*>(params);
  A.params16 = bf16 ? static_cast<uint16_t*>(params) : nullptr;
  A.grads = grads;
  A.codes = st + h->off_codes;
  A.window = reinterpret_cast<uint32_t*>(st + h->off_window);
  A.hdr = reinterpret_cast<uint32_t*>(st);
  A.mhat = mhat;
  A.vhat = vhat;
  A.row = (int32_t)(t % h->m);
  A.rows = (int32_t)std::min<int64_t>(t, h->m);
  A.pair_cur = pair_word(t);
  A.pair_next = pair_word(t + 1);
  A.t_lo = (uint32_t)(uint64_t)t;
  A.t_hi = (uint32_t)((uint64_t)t >> 32);
  const double b1 = beta1, b2 = beta2;
  A.lr = lr;
  A.eps = eps;
  A.decay = (float)(1.0 - (double)lr * (double)wd);
  A.has_decay = (wd != 0.0f);
  // Exact for e < 2^16: (2^32 mod kp) < kp and e * kp < 2^31 keep the error below 1/kp.
  A.kp_recip = (uint32_t)(((1ull << 32) + (uint64_t)h->kp - 1) / (uint64_t)h->kp);
  A.wait_ns = (uint64_t)std::max<int64_t>(0, h->wait_ns);
  A.n_seg = h->n_seg;
  for (int32_t s = 0; s < h->n_seg; ++s) {
    A.seg_first[s] = h->seg_first[s];
    A.seg_start[s] = h->seg_start[s];
    A.seg_len[s] = h->seg_len[s];
  }
  // Adam's bias correction of the unrolled sums [MicroAdam ¶1]:
  // m_hat = (1-beta1)/(1-beta1^t) * sum_r beta1^r V_r, likewise v_hat.
  A.f1 = (float)((1.0 - b1) / (1.0 - std::pow(b1, (double)t)));
  A.f2 = (float)((1.0 - b2) / (1.0 - std::pow(b2, (double)t)));
  for (int r = 0; r < h->m; ++r) {
    A.w1[r] = (float)std::pow(b1, (double)r);
    A.w2[r] = (float)std::pow(b2, (double)r);
  }
  uint32_t k0 = (uint32_t)seed, k1 = (uint32_t)(seed >> 32);
  for (int r = 0; r < 10; ++r) {  // Philox4x32-10 round keys (Salmon et al.)
    A.keys[r][0] = k0;
    A.keys[r][1] = k1;
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  return MUA_OK;
}

int mua_select(mua_t h, float* params, const uint16_t* grads, void* state, float lr,
               float beta1, float beta2, float eps, float wd, int64_t t, uint64_t seed,
               float* mhat, float* vhat, void* stream) {
  mua::StepArgs A;
  const int rc = fill_args(h, params, false, grads, state, lr, beta1, beta2, eps, wd, t, seed,
                           mhat, vhat, &A, /*params_optional=*/true);
  if (rc != MUA_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(A.hdr + A.pair_next, 0, 8, s);
  if (e != cudaSuccess) return cuda_fail(e, "reset of the min/max pair");
  e = mua::launch_select_warp(A, h->vec, s);
  if (e != cudaSuccess) return cuda_fail(e, "select kernel launch");
  return MUA_OK;
}

static int apply_impl(mua_t h, void* params, bool bf16, const uint16_t* grads, void* state,
                      float lr, float beta1, float beta2, float eps, float wd, int64_t t,
                      uint64_t seed, float* mhat, float* vhat, void* stream) {
  mua::StepArgs A;
  const int rc = fill_args(h, params, bf16, grads, state, lr, beta1, beta2, eps, wd, t, seed,
                           mhat, vhat, &A);
  if (rc != MUA_OK) return rc;
  const cudaError_t e = mua::launch_apply(A, h->apply_threads, h->vec, h->apply_smem,
                                          static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "apply kernel launch");
  return MUA_OK;
}

int mua_apply(mua_t h, float* params, const uint16_t* grads, void* state, float lr,
              float beta1, float beta2, float eps, float wd, int64_t t, uint64_t seed,
              float* mhat, float* vhat, void* stream) {
  return apply_impl(h, params, false, grads, state, lr, beta1, beta2, eps, wd, t, seed, mhat,
                    vhat, stream);
}

int mua_apply_bf16(mua_t h, uint16_t* params, const uint16_t* grads, void* state, float lr,
                   float beta1, float beta2, float eps, float wd, int64_t t, uint64_t seed,
                   float* mhat, float* vhat, void* stream) {
  return apply_impl(h, params, true, grads, state, lr, beta1, beta2, eps, wd, t, seed, mhat,
                    vhat, stream);
}

// Whether mua_step runs as one fused launch on the current device: a whole
// vector of blocks of at most 16384 entries, all of whose CTAs the device
// holds at once. Returns a negative MUA_ERR_CUDA code if the query fails.
static int use_fused(mua_t h, bool bf16) {
  if (!h->whole || h->Bd > 16384) return 0;
  int dev = 0;
  const cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "device query");
  const bool known = dev >= 0 && dev < mua::kMaxDevices;
  int cap = known ? h->fused_cap[bf16][dev] : -1;
  if (cap < 0) {
    cap = mua::fused_max_blocks(h->Bd, h->kp, h->m, h->vec, bf16);
    if (known) h->fused_cap[bf16][dev] = cap;
  }
  return h->nb <= cap ? 1 : 0;
}

static int step_impl(mua_t h, void* params, bool bf16, const uint16_t* grads, void* state,
                     float lr, float beta1, float beta2, float eps, float wd, int64_t t,
                     uint64_t seed, void* stream) {
  mua::StepArgs A;
  int rc = fill_args(h, params, bf16, grads, state, lr, beta1, beta2, eps, wd, t, seed, nullptr,
                     nullptr, &A);
  if (rc != MUA_OK) return rc;
  const int fused = use_fused(h, bf16);
  if (fused < 0) return fused;
  if (!fused) {
    rc = mua_select(h, nullptr, grads, state, lr, beta1, beta2, eps, wd, t, seed, nullptr,
                    nullptr, stream);
    if (rc != MUA_OK) return rc;
    return apply_impl(h, params, bf16, grads, state, lr, beta1, beta2, eps, wd, t, seed,
                      nullptr, nullptr, stream);
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(A.hdr + A.pair_next, 0, 8, s);
  if (e != cudaSuccess) return cuda_fail(e, "reset of the min/max pair");
  e = cudaMemsetAsync(A.hdr + mua::kHdrBarrier, 0, 4, s);
  if (e != cudaSuccess) return cuda_fail(e, "reset of the barrier word");
  e = mua::launch_fused(A, h->vec, s);
  if (e != cudaSuccess) return cuda_fail(e, "fused kernel launch");
  return MUA_OK;
}

int mua_step(mua_t h, float* params, const uint16_t* grads, void* state, float lr, float beta1,
             float beta2, float eps, float wd, int64_t t, uint64_t seed, void* stream) {
  return step_impl(h, params, false, grads, state, lr, beta1, beta2, eps, wd, t, seed, stream);
}

int mua_step_bf16(mua_t h, uint16_t* params, const uint16_t* grads, void* state, float lr,
                  float beta1, float beta2, float eps, float wd, int64_t t, uint64_t seed,
                  void* stream) {
  return step_impl(h, params, true, grads, state, lr, beta1, beta2, eps, wd, t, seed, stream);
}

int mua_step_launches(mua_t h, int32_t bf16_params) {
  if (!h) return MUA_ERR_ARG;
  const int fused = use_fused(h, bf16_params != 0);
  if (fused < 0) return fused;
  return fused ? 1 : 2;
}

int mua_set_wait_limit_ns(mua_t h, int64_t ns) {
  if (!h) return MUA_ERR_ARG;
  h->wait_ns = ns <= 0 ? 0 : ns;
  return MUA_OK;
}

int mua_get_status(mua_t h, const void* state, void* stream, int32_t* out) {
  if (!h || !state || !out) return MUA_ERR_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const uint32_t* hdr = static_cast<const uint32_t*>(state);
  cudaError_t e = cudaMemcpyAsync(out, hdr + mua::kHdrStatus, 4, cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return cuda_fail(e, "status copy");
  e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "status synchronize");
  return MUA_OK;
}

const char* mua_strerror(int code) {
  switch (code) {
    case MUA_OK: return "ok";
    case MUA_ERR_ARG: return "argument out of range or NULL";
    case MUA_ERR_UNSUPPORTED: return "unsupported configuration (bits != 4, window too large, odd tensor length or too many tensors)";
    case MUA_ERR_ALIGN: return "device pointer not 16-byte aligned";
    case MUA_ERR_CUDA: return "CUDA runtime error (see mua_last_cuda_error)";
    default: return "unknown error code";
  }
}

const char* mua_last_cuda_error(void) { return g_cuda_err; }

const char* mua_version(void) { return "mua 0.1 (sm_100a)"; }

}  // extern "C"
