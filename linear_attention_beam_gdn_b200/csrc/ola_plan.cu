// Depth-first beam order, part of the ancestry index.
//
// "Scientific Impact Assessment: OneLA", §1 Core Contribution: the ancestry index separates
// the logical evolution of beams (pruning, reordering, fan-out) from where their records
// live. Records stay where they were written; what this kernel adds is an ORDER in which a
// step visits the beams: depth-first over the beam tree, so that beams sharing ancestors are
// processed next to each other and their ancestors' records are read back to back (from L1
// and L2) instead of being scattered across the step.
//
// Step t (one CTA per request): key(b) = depth-first position of b's parent at step t-1
// (every key is 0 at step 1), and beams are stably sorted by key:
//     position(b) = #{b' : key(b') < key(b)} + #{b' < b : key(b') = key(b)}.
// Children of one parent become contiguous and parents keep their own depth-first order, so
// by induction the order is a depth-first order of the whole tree. Outputs: perm[r][pos] = b,
// pparent[r][pos] = parent of that beam, pchain[r][pos][:] = that parent's chain of record
// beam indices, and rank_cur[r][b] = pos (the next step's keys).
// Out-of-range parents are clamped to 0 and reported (OLA_ERR_BAD_PARENT), exactly as the
// decode kernels do.
#include <limits.h>

#include "ola_device.cuh"

namespace ola {

__global__ void __launch_bounds__(512) plan_kernel(StepArgs a) {
  extern __shared__ int keys[];                    // [Bp], Bp = B rounded up to 4
  const int r = blockIdx.x;
  const int B = a.B;
  const int Bp = (B + 3) & ~3;
  int* pbuf = keys + Bp;                           // [B] clamped parents
  for (int b = threadIdx.x; b < Bp; b += blockDim.x) {
    int key = INT_MAX;                             // padding sorts after every beam
    if (b < B) {
      const int p = checked_parent(a, r, b);
      key = (a.t == 1) ? 0 : a.rank_prev[size_t(r) * B + p];
      pbuf[b] = p;
    }
    keys[b] = key;
  }
  __syncthreads();
  const int4* k4 = reinterpret_cast<const int4*>(keys);
  for (int b = threadIdx.x; b < B; b += blockDim.x) {
    const int k = keys[b];
    int pos = 0;
    for (int j = 0; j < Bp / 4; ++j) {
      const int4 kk = k4[j];
      const int b2 = 4 * j;
      pos += (kk.x < k) | ((kk.x == k) & (b2 + 0 < b));
      pos += (kk.y < k) | ((kk.y == k) & (b2 + 1 < b));
      pos += (kk.z < k) | ((kk.z == k) & (b2 + 2 < b));
      pos += (kk.w < k) | ((kk.w == k) & (b2 + 3 < b));
    }
    a.perm[size_t(r) * B + pos] = b;
    a.pparent[size_t(r) * B + pos] = pbuf[b];
    a.rank_cur[size_t(r) * B + b] = pos;
    // the parent's chain, stored by position so a decode CTA reads it without first
    // resolving the beam and its parent
    if (a.pchain != nullptr)
      for (int s = 0; s < a.t - 1; ++s)
        a.pchain[(size_t(r) * B + pos) * a.T_max + s] = a.C[chain_row(a, a.t - 2, r, pbuf[b]) + s];
  }
}

cudaError_t launch_plan(const StepArgs& a, cudaStream_t stream) {
  const int Bp = (a.B + 3) & ~3;
  const int threads = a.B >= 512 ? 512 : ((a.B + 31) / 32) * 32;
  plan_kernel<<<a.R, threads, sizeof(int) * (Bp + a.B), stream>>>(a);
  return cudaGetLastError();
}

}  // namespace ola
