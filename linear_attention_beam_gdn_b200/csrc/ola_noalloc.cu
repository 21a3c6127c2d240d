// ola_decode_noalloc: a whole T-step decode that allocates no device memory.
//
// Who needs this: callers that may not call cudaMalloc while they decode. A server whose device
// memory is reserved up front by an arena or caching allocator cannot let a library take memory
// behind its back (a cudaMalloc could fail once the arena holds the device, or fragment it); a
// plugin loaded into a host application may be forbidden to allocate at all; a latency-critical
// decode loop cannot afford the device-wide synchronisation a cudaMalloc / cudaFree can imply.
// They pass every input and output buffer; the transient state of the decode (the transition
// records, the ancestry rows and the device error word) lives in one fixed array of this file,
// g_noalloc_scratch, which every GPU that loads the library holds until the process exits.
//
// The decode runs the CUDA-core fp32 replay kernel (ola_replay_simt.cu) once per step with its
// record pointers placed inside that array. The paper has no counterpart of this entry point.
#include <mutex>

#include "ola_device.cuh"

namespace ola {
cudaError_t launch_replay_simt(const StepArgs& a, int in_dtype, cudaStream_t stream);
size_t replay_simt_smem(int d_k, int d_v, int T_max);
ola_status validate_geometry(const ola_geometry* g);
}

using namespace ola;

// Fixed scratch shared by every call on a device (contents persist between calls).
static __device__ __align__(256) unsigned char g_noalloc_scratch[OLA_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mutex;

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Device address of the scratch array on the current device (resolved once per device).
cudaError_t scratch_address(unsigned char** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = static_cast<unsigned char*>(g_scratch_addr[dev]);
  return cudaSuccess;
}

}  // namespace

extern "C" {

uint64_t ola_noalloc_scratch_bytes(const ola_geometry* g) {
  if (!g || g->R < 1 || g->H < 1 || g->B < 1 || g->T_max < 1) return 0;
  const size_t R = g->R, H = g->H, B = g->B, T = g->T_max;
  const size_t e = g->in_dtype == OLA_BF16 ? 2 : 4;
  return 256 + align256(T * R * B * T * 4) + align256(T * R * H * B * 4) +
         align256(T * R * H * B * size_t(g->d_v) * 4) + align256(T * R * H * B * size_t(g->d_k) * e);
}

ola_status ola_decode_noalloc(const ola_geometry* g, const float* S_ctx, const void* q,
                              const void* k, const void* v, const float* gdec,
                              const float* beta, const int32_t* parent_idx, float* out_o,
                              void* stream) {
  // host-side checks first (no CUDA call before they pass): the geometry limits of ola_create
  // and the pointer rules of ola_create / ola_step
  ola_status vs = validate_geometry(g);
  if (vs != OLA_OK) return vs;
  if (g->path != OLA_PATH_REPLAY || g->math != OLA_MATH_FP32) return OLA_ERR_UNSUPPORTED;
  if (!S_ctx || !q || !k || !v || !gdec || !beta || !parent_idx || !out_o)
    return OLA_ERR_INVALID_ARG;
  if (!aligned(S_ctx, 16) || !aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) ||
      !aligned(out_o, 16) || !aligned(gdec, 4) || !aligned(beta, 4) || !aligned(parent_idx, 4))
    return OLA_ERR_INVALID_ARG;
  const uint64_t need = ola_noalloc_scratch_bytes(g);
  if (need > OLA_NOALLOC_SCRATCH_BYTES) return OLA_ERR_SCRATCH_LIMIT;
  // device checks (attribute queries only): an sm_100 device whose shared memory holds the
  // kernel's per-block footprint
  int dev = 0, major = 0, smem_optin = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
          cudaSuccess) {
    cudaGetLastError();
    return OLA_ERR_CUDA;
  }
  if (major != 10 || replay_simt_smem(g->d_k, g->d_v, g->T_max) > size_t(smem_optin))
    return OLA_ERR_UNSUPPORTED;

  unsigned char* base = nullptr;
  cudaError_t e = scratch_address(&base);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return OLA_ERR_CUDA;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t R = g->R, H = g->H, B = g->B, T = g->T_max;
  const size_t es = g->in_dtype == OLA_BF16 ? 2 : 4;
  int* err = reinterpret_cast<int*>(base);
  int* C = reinterpret_cast<int*>(base + 256);
  float* A = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(C) + align256(T * R * B * T * 4));
  float* W = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(A) + align256(T * R * H * B * 4));
  void* Kr = reinterpret_cast<unsigned char*>(W) + align256(T * R * H * B * size_t(g->d_v) * 4);

  // the error word is the only part that must start at zero
  e = cudaMemsetAsync(err, 0, 16, st);
  const size_t step_qk = R * B * H * size_t(g->d_k) * es;
  const size_t step_v = R * B * H * size_t(g->d_v) * es;
  const size_t step_s = R * B * H;
  for (int t = 1; e == cudaSuccess && t <= g->T_max; ++t) {
    StepArgs a{};
    a.R = g->R;
    a.H = g->H;
    a.d_k = g->d_k;
    a.d_v = g->d_v;
    a.B = g->B;
    a.T_max = g->T_max;
    a.t = t;
    a.q = static_cast<const unsigned char*>(q) + (t - 1) * step_qk;
    a.k = static_cast<const unsigned char*>(k) + (t - 1) * step_qk;
    a.v = static_cast<const unsigned char*>(v) + (t - 1) * step_v;
    a.g = gdec + (t - 1) * step_s;
    a.beta = beta + (t - 1) * step_s;
    a.parent = parent_idx + (t - 1) * R * B;
    a.o = out_o + (t - 1) * step_s * size_t(g->d_v);
    a.S = S_ctx;
    a.W = W;
    a.Kr = Kr;
    a.A = A;
    a.C = C;
    a.err = err;
    e = launch_replay_simt(a, g->in_dtype, st);
  }
  int word[4] = {0, 0, 0, 0};
  if (e == cudaSuccess) e = cudaMemcpyAsync(word, err, 16, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) {
    // a launch that failed part-way leaves the earlier steps queued: wait for them, so that
    // no kernel of this call still writes the scratch array once the call has returned
    cudaGetLastError();
    cudaStreamSynchronize(st);
    cudaGetLastError();
    return OLA_ERR_CUDA;
  }
  return static_cast<ola_status>(word[0]);
}

}  // extern "C"
