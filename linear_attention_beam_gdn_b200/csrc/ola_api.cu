// Host side of the C ABI declared in include/ola.h: argument validation, buffer ownership,
// kernel dispatch, the sticky device error word and the host-buffer entry point.
#include <stdint.h>
#include <string.h>

#include <new>

#include <algorithm>
#include <mutex>
#include <vector>

#include "ola_device.cuh"

namespace ola {
cudaError_t launch_prefill(int R, int H, int d_k, int d_v, int P, int in_dtype, const void* k,
                           const void* v, const float* g, const float* beta, float* S_out,
                           cudaStream_t stream);
bool prefill_chunk_supported(int d_k, int d_v, int in_dtype, const void* k, const void* v);
cudaError_t launch_prefill_chunk(int R, int H, int P, const void* k, const void* v,
                                 const float* g, const float* beta, float* S_out, int* err,
                                 cudaStream_t stream);
cudaError_t launch_fullstate(const StepArgs& a, int in_dtype, cudaStream_t stream);
cudaError_t launch_replayssm(const StepArgs& a, int in_dtype, cudaStream_t stream);
cudaError_t launch_replay_simt(const StepArgs& a, int in_dtype, cudaStream_t stream);
size_t replay_simt_smem(int d_k, int d_v, int T_max);
cudaError_t launch_replay_tc(const StepArgs& a, const CUtensorMap& mhi, const CUtensorMap& mlo,
                             cudaStream_t stream);
size_t replay_tc_smem(int d_k, int d_v, int B, int T_max);
cudaError_t launch_replay_pos(const StepArgs& a, const CUtensorMap& mhi, const CUtensorMap& mlo,
                              cudaStream_t stream);
size_t replay_pos_smem(int d_k, int d_v, int T_max);
bool replay_pos_supported(int d_k, int d_v);
bool make_state_map(CUtensorMap* map, const void* base, int RH, int d_k, int d_v);
bool replay_pipe_supported(int d_k, int d_v, int T_max);
size_t replay_pipe_smem(int d_k, int T_max);
cudaError_t launch_replay_pipe(const StepArgs& a, const void* S_hi, const void* S_lo,
                               cudaStream_t stream);
bool replay_mma_supported(int d_k, int d_v, int B, int T_max);
size_t replay_mma_smem(int d_k, int d_v);
int replay_mma_unit_records(int d_k, int d_v);
size_t plan_units_smem(int B, int T_max);
cudaError_t launch_replay_mma(const StepArgs& a, const UnitPlan& up, const void* S_hi,
                              const void* S_lo, const CUtensorMap& mkr, const CUtensorMap& mw,
                              cudaStream_t stream);
bool make_record_maps(CUtensorMap* mkr, CUtensorMap* mw, const void* Kr, const void* W,
                      uint64_t n_rec, int d_k, int d_v);
cudaError_t launch_split_state(const float* S, void* hi, void* lo, int RH, int d_k, int d_v,
                               cudaStream_t stream);
cudaError_t launch_common_prefix(const int* C, int R, int B, int T_max, int t, int* out,
                                 cudaStream_t stream);
cudaError_t launch_fold(float* S, const void* W, const void* Kr, int k_is_bf16, const float* A,
                        const float* Bt, const int* C, int R, int H, int d_k, int d_v, int B,
                        int T_max, int t, int c, int layout, cudaStream_t stream);
cudaError_t launch_chain_shift(int* C, int R, int B, int T_max, int t, int c, cudaStream_t stream);
}  // namespace ola

using namespace ola;

struct ola_ctx {
  ola_geometry g;
  int device;
  int t;
  int sticky;
  float* S = nullptr;
  void* S_hi = nullptr;
  void* S_lo = nullptr;
  float* W = nullptr;
  void* Kr = nullptr;
  float* A = nullptr;
  void* Vr = nullptr;        // history-replay path: v of every record
  float* Br = nullptr;       // history-replay path: beta of every record
  int* C = nullptr;
  float* FS[2] = {nullptr, nullptr};
  int* perm = nullptr;       // [2][R][B] depth-first order of the current step and the
                             // parent of the beam at each position (tensor path)
  int* rank = nullptr;       // [2][R][B] depth-first position of each beam, by step parity
  int* pchain = nullptr;     // [R][B][T_max] parent chain by depth-first position
  int* err = nullptr;
  int* lens = nullptr;       // [R] shared chain prefix of each request (ola_compact)
  CUtensorMap m_hi, m_lo;
  CUtensorMap m_kr, m_w;     // record row maps of the mma kernel
  bool pipe = false;         // tensor path on the persistent pipelined kernel
  bool mma = false;          // tensor path with the replay accumulation on tensor cores
  UnitPlan up{};             // units of work of the mma kernel (rewritten every step)
  // staging buffers of ola_step_host (allocated on first use)
  void* st[7] = {nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr};
  cudaStream_t last_stream = nullptr;
  // pipelined host-buffer steps (ola_step_host_async): two staging sets used alternately, a
  // copy-in and a copy-out stream, and the events that order them with the compute stream
  struct {
    void* buf[2][7] = {};
    cudaStream_t s_in = nullptr, s_out = nullptr;
    cudaEvent_t in_done[2] = {}, comp_done[2] = {}, out_done[2] = {};
    long long n = 0;                 // calls so far
  } hp;
};

namespace {

// Error word of the chunked prefill, one per device, allocated on first use and kept: a
// per-call stream-ordered allocation would map and unmap pool memory around every call.
constexpr int kMaxDevices = 64;
std::mutex g_prefill_mu;
int* g_prefill_err_dev[kMaxDevices] = {};
int* g_prefill_err_host[kMaxDevices] = {};

bool pow2_width(int d) { return d == 16 || d == 32 || d == 64 || d == 128 || d == 256; }
bool tc_width(int d) { return d == 64 || d == 128 || d == 256; }
bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

namespace ola {

// Host-side checks of a geometry shared by every entry point that takes one.
ola_status validate_geometry(const ola_geometry* g) {
  if (!g) return OLA_ERR_INVALID_ARG;
  if (g->R < 1 || g->H < 1 || g->B < 1 || g->T_max < 1) return OLA_ERR_INVALID_ARG;
  if (g->in_dtype != OLA_F32 && g->in_dtype != OLA_BF16) return OLA_ERR_INVALID_ARG;
  if (g->path != OLA_PATH_REPLAY && g->path != OLA_PATH_FULLSTATE &&
      g->path != OLA_PATH_REPLAYSSM)
    return OLA_ERR_INVALID_ARG;
  if (g->math != OLA_MATH_FP32 && g->math != OLA_MATH_TENSOR) return OLA_ERR_INVALID_ARG;
  if (!pow2_width(g->d_k) || !pow2_width(g->d_v)) return OLA_ERR_UNSUPPORTED;
  if (g->B > 4096 || g->T_max > 32) return OLA_ERR_UNSUPPORTED;
  if (int64_t(g->R) * g->H * g->B > (int64_t(1) << 30)) return OLA_ERR_UNSUPPORTED;
  if (g->math == OLA_MATH_TENSOR) {
    if (g->path != OLA_PATH_REPLAY || g->in_dtype != OLA_BF16) return OLA_ERR_UNSUPPORTED;
    if (!tc_width(g->d_k) || !tc_width(g->d_v)) return OLA_ERR_UNSUPPORTED;
    // record rows are 32-bit indices in the tensor-core kernel
    if (int64_t(g->T_max) * g->R * g->H * g->B >= (int64_t(1) << 31)) return OLA_ERR_UNSUPPORTED;
  }
  return OLA_OK;
}

}  // namespace ola

namespace {

ola_status validate(const ola_geometry* g) { return validate_geometry(g); }

struct Sizes {
  size_t S, S_split, W, Kr, A, Vr, Br, C, FS, perm, rank, pchain, err, lens;
  size_t ucnt, uoff, urec, upos, counter;   // mma path only
  size_t total() const {
    return S + 2 * S_split + W + Kr + A + Vr + Br + C + 2 * FS + perm + rank + pchain + err +
           lens + ucnt + uoff + urec + upos + counter;
  }
};

bool uses_mma(const ola_geometry* g) {
  return g->math == OLA_MATH_TENSOR && g->path == OLA_PATH_REPLAY &&
         replay_mma_supported(g->d_k, g->d_v, g->B, g->T_max);
}

Sizes sizes_of(const ola_geometry* g) {
  Sizes z{};
  const size_t R = g->R, H = g->H, B = g->B, T = g->T_max, dk = g->d_k, dv = g->d_v;
  const size_t e = g->in_dtype == OLA_BF16 ? 2 : 4;
  z.S = R * H * dv * dk * 4;
  z.S_split = g->math == OLA_MATH_TENSOR ? R * H * ((dv + 127) / 128 * 128) * dk * 2 : 0;
  const bool rep = g->path == OLA_PATH_REPLAY, rss = g->path == OLA_PATH_REPLAYSSM;
  z.W = rep ? T * R * H * B * dv * 4 : 0;
  z.Kr = (rep || rss) ? T * R * H * B * dk * e : 0;
  z.A = (rep || rss) ? T * R * H * B * 4 : 0;
  z.Vr = rss ? T * R * H * B * dv * e : 0;
  z.Br = rss ? T * R * H * B * 4 : 0;
  z.C = T * R * B * T * 4;
  z.FS = g->path == OLA_PATH_FULLSTATE ? R * H * B * dv * dk * 4 : 0;
  z.perm = g->math == OLA_MATH_TENSOR ? 2 * R * B * 4 : 0;
  z.rank = g->math == OLA_MATH_TENSOR ? 2 * R * B * 4 : 0;
  z.pchain = g->math == OLA_MATH_TENSOR ? R * B * T * 4 : 0;
  z.err = 16;
  z.lens = R * 4;
  if (uses_mma(g)) {
    z.ucnt = R * 4;
    z.uoff = (R + 1) * 4;
    z.urec = R * B * size_t(kUnitRecInts) * 4;   // at most B units per request
    z.upos = R * B * 16;
    z.counter = 16;
    z.pchain = 0;
  }
  return z;
}

ola_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return OLA_OK;
  cudaGetLastError();  // clear a non-sticky error
  return e == cudaErrorMemoryAllocation ? OLA_ERR_OOM : OLA_ERR_CUDA;
}

template <typename T>
cudaError_t dev_alloc(T** p, size_t bytes) {
  *p = nullptr;
  if (bytes == 0) return cudaSuccess;
  void* q = nullptr;
  cudaError_t e = cudaMalloc(&q, bytes);
  if (e == cudaSuccess) *p = static_cast<T*>(q);
  return e;
}

void free_all(ola_ctx* h) {
  void* ptrs[] = {h->S,     h->S_hi,  h->S_lo,   h->W,       h->Kr,     h->A,  h->Vr, h->Br,
                  h->C,     h->FS[0], h->FS[1],  h->perm,    h->rank,   h->pchain,
                  h->err,   h->lens,  h->up.ucnt, h->up.uoff, h->up.urec, h->up.upos,
                  h->up.counter};
  for (void* p : ptrs)
    if (p) cudaFree(p);
  for (void* p : h->st)
    if (p) cudaFree(p);
  for (auto& set : h->hp.buf)
    for (void* p : set)
      if (p) cudaFree(p);
  for (int i = 0; i < 2; ++i) {
    if (h->hp.in_done[i]) cudaEventDestroy(h->hp.in_done[i]);
    if (h->hp.comp_done[i]) cudaEventDestroy(h->hp.comp_done[i]);
    if (h->hp.out_done[i]) cudaEventDestroy(h->hp.out_done[i]);
  }
  if (h->hp.s_in) cudaStreamDestroy(h->hp.s_in);
  if (h->hp.s_out) cudaStreamDestroy(h->hp.s_out);
}

StepArgs make_args(ola_ctx* h, const void* q, const void* k, const void* v, const float* g,
                   const float* beta, const int32_t* parent, float* out_o) {
  StepArgs a;
  a.R = h->g.R;
  a.H = h->g.H;
  a.d_k = h->g.d_k;
  a.d_v = h->g.d_v;
  a.B = h->g.B;
  a.T_max = h->g.T_max;
  a.t = h->t + 1;
  a.q = q;
  a.k = k;
  a.v = v;
  a.g = g;
  a.beta = beta;
  a.parent = parent;
  a.o = out_o;
  a.S = h->S;
  a.W = h->W;
  a.Kr = h->Kr;
  a.A = h->A;
  a.C = h->C;
  a.FS_prev = h->FS[(a.t + 1) & 1];   // states of step t-1 (unused at t = 1)
  a.FS_cur = h->FS[a.t & 1];
  const size_t RB = size_t(h->g.R) * h->g.B;
  a.perm = h->perm;
  a.pparent = h->perm ? h->perm + RB : nullptr;
  a.pchain = h->pchain;
  a.rank_prev = h->rank ? h->rank + ((a.t + 1) & 1) * RB : nullptr;
  a.rank_cur = h->rank ? h->rank + (a.t & 1) * RB : nullptr;
  a.err = h->err;
  a.Vr = h->Vr;
  a.Br = h->Br;
  return a;
}

}  // namespace

extern "C" {

int32_t ola_version(void) { return (1 << 16) | 0; }

const char* ola_strerror(ola_status s) {
  switch (s) {
    case OLA_OK: return "ok";
    case OLA_ERR_INVALID_ARG: return "invalid argument";
    case OLA_ERR_UNSUPPORTED: return "unsupported geometry or device";
    case OLA_ERR_CAPACITY: return "step capacity T_max exhausted";
    case OLA_ERR_BAD_PARENT: return "parent index out of range";
    case OLA_ERR_OOM: return "device out of memory";
    case OLA_ERR_CUDA: return "CUDA runtime error";
    case OLA_ERR_TIMEOUT: return "bounded device wait timed out";
    case OLA_ERR_SCRATCH_LIMIT: return "problem exceeds the fixed no-allocation scratch";
  }
  return "unknown status";
}

ola_status ola_workspace_bytes(const ola_geometry* geom, uint64_t* out_bytes) {
  if (!out_bytes) return OLA_ERR_INVALID_ARG;
  ola_status s = validate(geom);
  if (s != OLA_OK) return s;
  *out_bytes = sizes_of(geom).total();
  return OLA_OK;
}

ola_status ola_create(const ola_geometry* geom, const float* S_ctx, void* stream,
                      ola_handle* out) {
  if (!out) return OLA_ERR_INVALID_ARG;
  *out = nullptr;
  ola_status s = validate(geom);
  if (s != OLA_OK) return s;
  if (!S_ctx || !aligned(S_ctx, 16)) return OLA_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return from_cuda(cudaGetLastError());
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return OLA_ERR_CUDA;
  if (prop.major != 10) return OLA_ERR_UNSUPPORTED;
  if (geom->path == OLA_PATH_REPLAY) {
    size_t smem = geom->math != OLA_MATH_TENSOR
                      ? replay_simt_smem(geom->d_k, geom->d_v, geom->T_max)
                  : uses_mma(geom) ? replay_mma_smem(geom->d_k, geom->d_v)
                  : replay_pipe_supported(geom->d_k, geom->d_v, geom->T_max)
                      ? replay_pipe_smem(geom->d_k, geom->T_max)
                  : replay_pos_supported(geom->d_k, geom->d_v)
                      ? replay_pos_smem(geom->d_k, geom->d_v, geom->T_max)
                      : replay_tc_smem(geom->d_k, geom->d_v, geom->B, geom->T_max);
    if (smem > size_t(prop.sharedMemPerBlockOptin)) return OLA_ERR_UNSUPPORTED;
    if (uses_mma(geom) &&
        plan_units_smem(geom->B, geom->T_max) > size_t(prop.sharedMemPerBlockOptin))
      return OLA_ERR_UNSUPPORTED;
  }

  ola_ctx* h = new (std::nothrow) ola_ctx();
  if (!h) return OLA_ERR_OOM;
  h->g = *geom;
  h->device = dev;
  h->t = 0;
  h->sticky = 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  h->last_stream = st;
  const Sizes z = sizes_of(geom);
  cudaError_t e = cudaSuccess;
  if (e == cudaSuccess) e = dev_alloc(&h->S, z.S);
  if (e == cudaSuccess) e = dev_alloc(&h->S_hi, z.S_split);
  if (e == cudaSuccess) e = dev_alloc(&h->S_lo, z.S_split);
  if (e == cudaSuccess) e = dev_alloc(&h->W, z.W);
  if (e == cudaSuccess) e = dev_alloc(&h->Kr, z.Kr);
  if (e == cudaSuccess) e = dev_alloc(&h->A, z.A);
  if (e == cudaSuccess) e = dev_alloc(&h->Vr, z.Vr);
  if (e == cudaSuccess) e = dev_alloc(&h->Br, z.Br);
  if (e == cudaSuccess) e = dev_alloc(&h->C, z.C);
  if (e == cudaSuccess) e = dev_alloc(&h->FS[0], z.FS);
  if (e == cudaSuccess) e = dev_alloc(&h->FS[1], z.FS);
  if (e == cudaSuccess) e = dev_alloc(&h->perm, z.perm);
  if (e == cudaSuccess) e = dev_alloc(&h->rank, z.rank);
  if (e == cudaSuccess) e = dev_alloc(&h->pchain, z.pchain);
  if (e == cudaSuccess) e = dev_alloc(&h->err, z.err);
  if (e == cudaSuccess) e = dev_alloc(&h->lens, z.lens);
  if (e == cudaSuccess) e = dev_alloc(&h->up.ucnt, z.ucnt);
  if (e == cudaSuccess) e = dev_alloc(&h->up.uoff, z.uoff);
  if (e == cudaSuccess) e = dev_alloc(&h->up.urec, z.urec);
  if (e == cudaSuccess) e = dev_alloc(&h->up.upos, z.upos);
  if (e == cudaSuccess) e = dev_alloc(&h->up.counter, z.counter);
  if (e == cudaSuccess && z.counter) e = cudaMemsetAsync(h->up.counter, 0, z.counter, st);
  h->up.maxU = geom->B;
  h->up.maxAnc = replay_mma_unit_records(geom->d_k, geom->d_v);
  if (e == cudaSuccess) e = cudaMemcpyAsync(h->S, S_ctx, z.S, cudaMemcpyDeviceToDevice, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(h->err, 0, z.err, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(h->C, 0, z.C, st);
  if (e == cudaSuccess && geom->math == OLA_MATH_TENSOR) {
    const int RH = geom->R * geom->H;
    e = launch_split_state(h->S, h->S_hi, h->S_lo, RH, geom->d_k, geom->d_v, st);
    if (e == cudaSuccess && (!make_state_map(&h->m_hi, h->S_hi, RH, geom->d_k, geom->d_v) ||
                             !make_state_map(&h->m_lo, h->S_lo, RH, geom->d_k, geom->d_v)))
      e = cudaErrorInvalidValue;
    h->mma = uses_mma(geom);
    h->pipe = !h->mma && replay_pipe_supported(geom->d_k, geom->d_v, geom->T_max);
    const uint64_t n_rec = uint64_t(geom->T_max) * geom->R * geom->H * geom->B;
    if (e == cudaSuccess && h->mma &&
        !make_record_maps(&h->m_kr, &h->m_w, h->Kr, h->W, n_rec, geom->d_k, geom->d_v))
      e = cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) {
    ola_status rs = from_cuda(e);
    cudaStreamSynchronize(st);
    free_all(h);
    delete h;
    return rs;
  }
  *out = h;
  return OLA_OK;
}

ola_status ola_step(ola_handle h, const void* q, const void* k, const void* v, const float* g,
                    const float* beta, const int32_t* parent_idx, float* out_o, void* stream) {
  if (!h) return OLA_ERR_INVALID_ARG;
  if (!q || !k || !v || !g || !beta || !parent_idx || !out_o) return OLA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out_o, 16) ||
      !aligned(g, 4) || !aligned(beta, 4) || !aligned(parent_idx, 4))
    return OLA_ERR_INVALID_ARG;
  if (h->sticky) return static_cast<ola_status>(h->sticky);
  if (h->t >= h->g.T_max) return OLA_ERR_CAPACITY;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  StepArgs a = make_args(h, q, k, v, g, beta, parent_idx, out_o);
  cudaError_t e;
  if (h->g.path == OLA_PATH_FULLSTATE)
    e = launch_fullstate(a, h->g.in_dtype, st);
  else if (h->g.path == OLA_PATH_REPLAYSSM)
    e = launch_replayssm(a, h->g.in_dtype, st);
  else if (h->g.math == OLA_MATH_TENSOR && h->mma)
    e = launch_replay_mma(a, h->up, h->S_hi, h->S_lo, h->m_kr, h->m_w, st);
  else if (h->g.math == OLA_MATH_TENSOR && h->pipe)
    e = launch_replay_pipe(a, h->S_hi, h->S_lo, st);
  else if (h->g.math == OLA_MATH_TENSOR && replay_pos_supported(h->g.d_k, h->g.d_v))
    e = launch_replay_pos(a, h->m_hi, h->m_lo, st);
  else if (h->g.math == OLA_MATH_TENSOR)
    e = launch_replay_tc(a, h->m_hi, h->m_lo, st);
  else
    e = launch_replay_simt(a, h->g.in_dtype, st);
  if (e != cudaSuccess) return from_cuda(e);
  h->t += 1;
  h->last_stream = st;
  return OLA_OK;
}

ola_status ola_step_host(ola_handle h, const void* q, const void* k, const void* v,
                         const float* g, const float* beta, const int32_t* parent_idx,
                         float* out_o, void* stream) {
  if (!h) return OLA_ERR_INVALID_ARG;
  if (!q || !k || !v || !g || !beta || !parent_idx || !out_o) return OLA_ERR_INVALID_ARG;
  const size_t R = h->g.R, B = h->g.B, H = h->g.H;
  const size_t e = h->g.in_dtype == OLA_BF16 ? 2 : 4;
  const size_t bytes[7] = {R * B * H * h->g.d_k * e, R * B * H * h->g.d_k * e,
                           R * B * H * h->g.d_v * e, R * B * H * 4, R * B * H * 4, R * B * 4,
                           R * B * H * h->g.d_v * 4};
  for (int i = 0; i < 7; ++i)
    if (!h->st[i]) {
      cudaError_t ce = cudaMalloc(&h->st[i], bytes[i]);
      if (ce != cudaSuccess) return from_cuda(ce);
    }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const void* src[6] = {q, k, v, g, beta, parent_idx};
  for (int i = 0; i < 6; ++i) {
    cudaError_t ce = cudaMemcpyAsync(h->st[i], src[i], bytes[i], cudaMemcpyHostToDevice, st);
    if (ce != cudaSuccess) return from_cuda(ce);
  }
  ola_status s = ola_step(h, h->st[0], h->st[1], h->st[2], static_cast<const float*>(h->st[3]),
                          static_cast<const float*>(h->st[4]),
                          static_cast<const int32_t*>(h->st[5]), static_cast<float*>(h->st[6]),
                          stream);
  if (s != OLA_OK) return s;
  cudaError_t ce = cudaMemcpyAsync(out_o, h->st[6], bytes[6], cudaMemcpyDeviceToHost, st);
  if (ce != cudaSuccess) return from_cuda(ce);
  return from_cuda(cudaStreamSynchronize(st));
}

ola_status ola_step_host_async(ola_handle h, const void* q, const void* k, const void* v,
                               const float* g, const float* beta, const int32_t* parent_idx,
                               float* out_o, void* stream) {
  if (!h) return OLA_ERR_INVALID_ARG;
  if (!q || !k || !v || !g || !beta || !parent_idx || !out_o) return OLA_ERR_INVALID_ARG;
  auto& hp = h->hp;
  const size_t R = h->g.R, B = h->g.B, H = h->g.H;
  const size_t e = h->g.in_dtype == OLA_BF16 ? 2 : 4;
  const size_t bytes[7] = {R * B * H * h->g.d_k * e, R * B * H * h->g.d_k * e,
                           R * B * H * h->g.d_v * e, R * B * H * 4, R * B * H * 4, R * B * 4,
                           R * B * H * h->g.d_v * 4};
  cudaError_t ce = cudaSuccess;
  if (!hp.s_in) {
    ce = cudaStreamCreateWithFlags(&hp.s_in, cudaStreamNonBlocking);
    if (ce == cudaSuccess) ce = cudaStreamCreateWithFlags(&hp.s_out, cudaStreamNonBlocking);
    for (int i = 0; i < 2 && ce == cudaSuccess; ++i) {
      ce = cudaEventCreateWithFlags(&hp.in_done[i], cudaEventDisableTiming);
      if (ce == cudaSuccess) ce = cudaEventCreateWithFlags(&hp.comp_done[i], cudaEventDisableTiming);
      if (ce == cudaSuccess) ce = cudaEventCreateWithFlags(&hp.out_done[i], cudaEventDisableTiming);
      for (int j = 0; j < 7 && ce == cudaSuccess; ++j) ce = cudaMalloc(&hp.buf[i][j], bytes[j]);
    }
    if (ce != cudaSuccess) return from_cuda(ce);
  }
  const int p = int(hp.n & 1);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  // copy-in: staging set p is free once the step of two calls ago has run
  if (hp.n >= 2) ce = cudaStreamWaitEvent(hp.s_in, hp.comp_done[p], 0);
  const void* src[6] = {q, k, v, g, beta, parent_idx};
  for (int i = 0; i < 6 && ce == cudaSuccess; ++i)
    ce = cudaMemcpyAsync(hp.buf[p][i], src[i], bytes[i], cudaMemcpyHostToDevice, hp.s_in);
  if (ce == cudaSuccess) ce = cudaEventRecord(hp.in_done[p], hp.s_in);
  // the step, on the caller's stream, after its inputs and after o of two calls ago is out
  if (ce == cudaSuccess) ce = cudaStreamWaitEvent(cs, hp.in_done[p], 0);
  if (ce == cudaSuccess && hp.n >= 2) ce = cudaStreamWaitEvent(cs, hp.out_done[p], 0);
  if (ce != cudaSuccess) return from_cuda(ce);
  ola_status s = ola_step(h, hp.buf[p][0], hp.buf[p][1], hp.buf[p][2],
                          static_cast<const float*>(hp.buf[p][3]),
                          static_cast<const float*>(hp.buf[p][4]),
                          static_cast<const int32_t*>(hp.buf[p][5]),
                          static_cast<float*>(hp.buf[p][6]), stream);
  if (s != OLA_OK) return s;
  // copy-out, overlapping the next call's copy-in (the link carries both directions at once)
  ce = cudaEventRecord(hp.comp_done[p], cs);
  if (ce == cudaSuccess) ce = cudaStreamWaitEvent(hp.s_out, hp.comp_done[p], 0);
  if (ce == cudaSuccess)
    ce = cudaMemcpyAsync(out_o, hp.buf[p][6], bytes[6], cudaMemcpyDeviceToHost, hp.s_out);
  if (ce == cudaSuccess) ce = cudaEventRecord(hp.out_done[p], hp.s_out);
  if (ce != cudaSuccess) return from_cuda(ce);
  ++hp.n;
  return OLA_OK;
}

ola_status ola_host_sync(ola_handle h) {
  if (!h) return OLA_ERR_INVALID_ARG;
  if (h->hp.s_out) {
    cudaError_t ce = cudaStreamSynchronize(h->hp.s_in);
    if (ce == cudaSuccess) ce = cudaStreamSynchronize(h->hp.s_out);
    if (ce != cudaSuccess) return from_cuda(ce);
  }
  return ola_get_error(h);
}

ola_status ola_reset(ola_handle h) {
  if (!h) return OLA_ERR_INVALID_ARG;
  cudaError_t e = cudaMemsetAsync(h->err, 0, 16, h->last_stream);
  if (e != cudaSuccess) return from_cuda(e);
  h->t = 0;
  h->sticky = 0;
  return OLA_OK;
}

ola_status ola_compact(ola_handle h, int32_t* out_folded, void* stream) {
  if (!h) return OLA_ERR_INVALID_ARG;
  if (out_folded) *out_folded = 0;
  if (h->sticky) return static_cast<ola_status>(h->sticky);
  const ola_geometry& g = h->g;
  const int t = h->t;
  if (t < 2) return OLA_OK;   // nothing to fold
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  h->last_stream = st;
  // shared chain prefix of every request (into the handle's own buffer: nothing is allocated)
  cudaError_t e = launch_common_prefix(h->C, g.R, g.B, g.T_max, t, h->lens, st);
  std::vector<int> host(size_t(g.R), 0);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(host.data(), h->lens, size_t(g.R) * 4, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return from_cuda(e);
  int c = t - 1;
  for (int x : host) c = std::min(c, x);
  if (c <= 0) return OLA_OK;
  if (g.path == OLA_PATH_FULLSTATE) {
    // the beams' states are materialised and hold every step: only the ancestry rows of the
    // shared slots are dropped; the state buffers follow the parity of the lowered step count
    e = launch_chain_shift(h->C, g.R, g.B, g.T_max, t, c, st);
    if (e != cudaSuccess) return from_cuda(e);
    if (c & 1) std::swap(h->FS[0], h->FS[1]);
    h->t = t - c;
    if (out_folded) *out_folded = c;
    return OLA_OK;
  }
  // fold the shared records into S_ctx (and its bf16 split), then move the later record slots
  // and the chain rows down by c
  const bool rss = g.path == OLA_PATH_REPLAYSSM;
  const int layout = rss ? 2 : h->mma ? 1 : 0;
  e = launch_fold(h->S, rss ? h->Vr : h->W, h->Kr, g.in_dtype == OLA_BF16, h->A, h->Br, h->C,
                  g.R, g.H, g.d_k, g.d_v, g.B, g.T_max, t, c, layout, st);
  if (e == cudaSuccess && g.math == OLA_MATH_TENSOR)
    e = launch_split_state(h->S, h->S_hi, h->S_lo, g.R * g.H, g.d_k, g.d_v, st);
  const size_t rows = size_t(g.R) * g.H * g.B;
  const size_t kbytes = g.in_dtype == OLA_BF16 ? 2 : 4;
  // per record slot: w (or, on the history-replay path, v and beta), k, alpha
  const size_t w_slot = rss ? rows * g.d_v * kbytes : rows * g.d_v * 4;
  const size_t k_slot = rows * g.d_k * kbytes, a_slot = rows * 4;
  char* const bufs[4] = {reinterpret_cast<char*>(rss ? h->Vr : h->W), static_cast<char*>(h->Kr),
                         reinterpret_cast<char*>(h->A), reinterpret_cast<char*>(h->Br)};
  const size_t slot_bytes[4] = {w_slot, k_slot, a_slot, rss ? a_slot : 0};
  for (int s = c; s < t && e == cudaSuccess; ++s)     // increasing order: sources stay intact
    for (int x = 0; x < 4 && e == cudaSuccess; ++x)
      if (slot_bytes[x])
        e = cudaMemcpyAsync(bufs[x] + (s - c) * slot_bytes[x], bufs[x] + s * slot_bytes[x],
                            slot_bytes[x], cudaMemcpyDeviceToDevice, st);
  if (e == cudaSuccess) e = launch_chain_shift(h->C, g.R, g.B, g.T_max, t, c, st);
  // the next step reads the depth-first ranks of this one from the buffer of its parity
  const size_t RB = size_t(g.R) * g.B;
  if (e == cudaSuccess && h->rank && (c & 1))
    e = cudaMemcpyAsync(h->rank + size_t((t - c) & 1) * RB, h->rank + size_t(t & 1) * RB, RB * 4,
                        cudaMemcpyDeviceToDevice, st);
  if (e != cudaSuccess) return from_cuda(e);
  h->t = t - c;
  if (out_folded) *out_folded = c;
  return OLA_OK;
}

int32_t ola_current_step(ola_handle h) { return h ? h->t : -1; }

ola_status ola_get_ancestry(ola_handle h, int32_t* out, void* stream) {
  if (!h || !out || h->t == 0) return OLA_ERR_INVALID_ARG;
  const size_t t = h->t, Tm = h->g.T_max;
  const int32_t* src = h->C + size_t(t - 1) * h->g.R * h->g.B * Tm;
  cudaError_t e = cudaMemcpy2DAsync(out, t * 4, src, Tm * 4, t * 4, size_t(h->g.R) * h->g.B,
                                    cudaMemcpyDeviceToDevice, static_cast<cudaStream_t>(stream));
  return from_cuda(e);
}

ola_status ola_get_error(ola_handle h) {
  if (!h) return OLA_ERR_INVALID_ARG;
  cudaError_t e = cudaStreamSynchronize(h->last_stream);
  if (e != cudaSuccess) return from_cuda(e);
  int w[4] = {0, 0, 0, 0};
  e = cudaMemcpy(w, h->err, 16, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return from_cuda(e);
  if (w[0] != 0) h->sticky = w[0];
  return static_cast<ola_status>(h->sticky);
}

ola_status ola_destroy(ola_handle h) {
  if (!h) return OLA_OK;
  cudaStreamSynchronize(h->last_stream);
  if (h->hp.s_out) {
    cudaStreamSynchronize(h->hp.s_in);
    cudaStreamSynchronize(h->hp.s_out);
  }
  free_all(h);
  delete h;
  return OLA_OK;
}

ola_status ola_prefill(int32_t R, int32_t H, int32_t d_k, int32_t d_v, int32_t P,
                       int32_t in_dtype, const void* k, const void* v, const float* g,
                       const float* beta, float* S_out, void* stream) {
  if (R < 1 || H < 1 || P < 0) return OLA_ERR_INVALID_ARG;
  if (in_dtype != OLA_F32 && in_dtype != OLA_BF16) return OLA_ERR_INVALID_ARG;
  if (!pow2_width(d_k) || !pow2_width(d_v)) return OLA_ERR_UNSUPPORTED;
  if (!S_out || !aligned(S_out, 16)) return OLA_ERR_INVALID_ARG;
  if (P > 0 && (!k || !v || !g || !beta)) return OLA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (P > 0 && prefill_chunk_supported(d_k, d_v, in_dtype, k, v)) {
    // chunked tensor-core form; waits for it so that a device-side timeout is returned
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return OLA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_prefill_mu);
    if (!g_prefill_err_dev[dev] || !g_prefill_err_host[dev]) {
      int* d = nullptr;
      int* hh = nullptr;
      if (cudaMalloc(reinterpret_cast<void**>(&d), 4 * sizeof(int)) != cudaSuccess)
        return OLA_ERR_OOM;
      if (cudaMallocHost(reinterpret_cast<void**>(&hh), 4 * sizeof(int)) != cudaSuccess) {
        cudaFree(d);
        return OLA_ERR_OOM;
      }
      g_prefill_err_dev[dev] = d;
      g_prefill_err_host[dev] = hh;
    }
    int* derr = g_prefill_err_dev[dev];
    int* herr = g_prefill_err_host[dev];
    cudaError_t e = cudaMemsetAsync(derr, 0, 4 * sizeof(int), st);
    if (e == cudaSuccess) e = launch_prefill_chunk(R, H, P, k, v, g, beta, S_out, derr, st);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(herr, derr, 4 * sizeof(int), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return from_cuda(e);
    return herr[0] != 0 ? static_cast<ola_status>(herr[0]) : OLA_OK;
  }
  return from_cuda(launch_prefill(R, H, d_k, d_v, P, in_dtype, k, v, g, beta, S_out, st));
}

}  // extern "C"
