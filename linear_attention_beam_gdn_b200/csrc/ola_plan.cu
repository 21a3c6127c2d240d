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

// ---------------------------------------------------------------------- units of work

// Depth-first positions cut into units for the tensor-core replay kernel (ola_replay_mma.cu).
//
// A unit is a run of at most kUnitPos consecutive depth-first positions of one request whose
// parent chains reach at most up.maxAnc distinct records. In depth-first order every record's
// descendants are contiguous, so within a chain slot the records of consecutive positions are
// equal or new, and the distinct records of a unit are the slot-wise changes. Units are made of
// whole sibling groups where they fit (see the cut below).
//
// For every unit the kernel writes one record of kUnitRecInts ints:
//   [0] start | n_pos << 16, [1] U (distinct records), [4 + p] beam at position start + p,
//   [36 + u] (slot << 16) | beam of distinct record u (slot order, then position order),
// and for every position p, upos[r][p][s] = index u of the record in chain slot s. It also
// writes the chain rows of the new beams (C[t-1][r][b] = parent's chain, then b), the number
// of units of each request and, in the last CTA to finish, their exclusive prefix sum.
size_t plan_units_smem(int B, int T_max) {
  const int Bp = (B + 3) & ~3, TA = T_max > 1 ? T_max - 1 : 1;
  // keys, parents, perm, chains, change masks, unit of position, unit start/size/U, counts,
  // sibling-group starts and sizes, prefix sums of group sizes and new-record counts, unit
  // ends, per-chunk key counts of the sort (16 x B uint16), per-position record indices
  // (B x 16 bytes), scratch
  return sizeof(int) * (size_t(Bp) + B + B + size_t(B) * TA + B + B + 3 * size_t(B) +
                        size_t(B) * TA + 2 * size_t(B) + 3 * size_t(B + 1) + 8 * size_t(B) +
                        4 * size_t(B) + 4 + 128);
}

__global__ void __launch_bounds__(512) plan_units_kernel(StepArgs a, UnitPlan up) {
  extern __shared__ int sm[];
  const int r = blockIdx.x, B = a.B, Bp = (B + 3) & ~3;
  const int n_anc = a.t - 1, TA = a.T_max > 1 ? a.T_max - 1 : 1;
  const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, warp = tid >> 5;
  int* keys = sm;                 // [Bp]
  int* pbuf = keys + Bp;          // [B] clamped parent of beam b
  int* sperm = pbuf + B;          // [B] beam at position
  int* spch = sperm + B;          // [B][TA] parent chain by position
  int* fnew = spch + B * TA;      // [B] slots where the record differs from the position before
  int* uop = fnew + B;            // [B] unit of position
  int* ustart = uop + B;          // [B]
  int* un = ustart + B;           // [B]
  int* uU = un + B;               // [B]
  int* sdist = uU + B;            // [B][TA] distinct records per (unit, slot)
  int* gst = sdist + B * TA;      // [B] start of each sibling group
  int* gsz = gst + B;             // [B] its size
  int* PS = gsz + B;              // [B + 1] prefix sums of the group sizes
  int* PC = PS + (B + 1);         // [B + 1] prefix sums of the groups' new-record counts
  int* gnext = PC + (B + 1);      // [B + 1] end (exclusive) of a unit starting at group g
  unsigned short* ccnt = reinterpret_cast<unsigned short*>(gnext + (B + 1));   // [16][B]
  int* upos_i = gnext + (B + 1) + 8 * B;
  upos_i += (4 - (reinterpret_cast<uintptr_t>(upos_i) >> 2) % 4) % 4;           // 16-byte aligned
  uint8_t* upos_s = reinterpret_cast<uint8_t*>(upos_i);                        // [B][16]
  int* misc = upos_i + 4 * B;     // [0] unit count, [1] last-CTA flag, [2] groups, [32..] scratch

  // depth-first order: stable sort of the beams by their parent's position (ola_plan.cu above)
  for (int b = tid; b < Bp; b += nt) {
    int key = INT_MAX;
    if (b < B) {
      const int p = checked_parent(a, r, b);
      key = (a.t == 1) ? 0 : a.rank_prev[size_t(r) * B + p];
      pbuf[b] = p;
    }
    keys[b] = key;
  }
  __syncthreads();
  if (B <= 512 && nt == 512) {
    // counting sort, stable: a warp per chunk of 32 beams finds the beams of its chunk with
    // equal keys (match), per key the counts of the earlier chunks are summed, and the key
    // offsets come from a scan; position = beams with a smaller key + beams with the same key
    // in earlier chunks + those earlier in this chunk
    int* off = ustart;                              // [B] (free until the unit cut)
    for (int x = tid; x < 16 * B; x += nt) ccnt[x] = 0;
    __syncthreads();
    const int b = 32 * warp + lane;
    const bool valid = b < B;
    const int k = valid ? keys[b] : -1 - lane;
    const unsigned peers = __match_any_sync(kFull, k);
    const int rin = __popc(peers & ((1u << lane) - 1u));
    if (valid && lane == __ffs(peers) - 1) ccnt[warp * B + k] = (unsigned short)__popc(peers);
    __syncthreads();
    for (int kk = tid; kk < B; kk += nt) {
      int run = 0;
      for (int j = 0; j < 16; ++j) {
        const int c = ccnt[j * B + kk];
        ccnt[j * B + kk] = (unsigned short)run;
        run += c;
      }
      off[kk] = run;                                // beams with key kk
    }
    __syncthreads();
    {                                               // exclusive scan of off over the keys
      const int v = tid < B ? off[tid] : 0;
      int x = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(kFull, x, o);
        if (lane >= o) x += y;
      }
      if (lane == 31) misc[32 + warp] = x;
      __syncthreads();
      int before = 0;
      for (int w2 = 0; w2 < warp; ++w2) before += misc[32 + w2];
      if (tid < B) off[tid] = before + x - v;
      __syncthreads();
    }
    if (valid) {
      const int pos = off[k] + ccnt[warp * B + k] + rin;
      a.perm[size_t(r) * B + pos] = b;
      a.rank_cur[size_t(r) * B + b] = pos;
      sperm[pos] = b;
    }
  } else {
    const int4* k4 = reinterpret_cast<const int4*>(keys);
    for (int b = tid; b < B; b += nt) {
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
      a.rank_cur[size_t(r) * B + b] = pos;
      sperm[pos] = b;
    }
  }
  __syncthreads();
  // parent chains by position; chain rows of the new beams (a thread per position: the parent's
  // chain entries are all loaded before any is stored)
  for (int pos = tid; pos < B; pos += nt) {
    const int b = sperm[pos];
    int* dst = a.C + chain_row(a, a.t - 1, r, b);
    for (int s0 = 0; s0 < n_anc; s0 += 8) {
      const int* src = a.C + chain_row(a, a.t - 2, r, pbuf[b]) + s0;
      int cv[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) cv[q] = s0 + q < n_anc ? src[q] : 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (s0 + q < n_anc) {
          spch[pos * TA + s0 + q] = cv[q];
          dst[s0 + q] = cv[q];
        }
      }
    }
    dst[n_anc] = b;
  }
  __syncthreads();
  for (int pos = tid; pos < B; pos += nt) {
    int m = 0;
    for (int s = 0; s < n_anc; ++s)
      if (pos == 0 || spch[pos * TA + s] != spch[(pos - 1) * TA + s]) m |= 1 << s;
    fnew[pos] = m;
  }
  __syncthreads();
  // sibling groups (runs of positions with the same parent): numbered by a block-wide scan
  {
    int carry = 0;
    for (int base = 0; base < B; base += nt) {
      const int pos = base + tid;
      const int f = (pos < B && (pos == 0 || keys[sperm[pos]] != keys[sperm[pos - 1]])) ? 1 : 0;
      int x = f;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(kFull, x, off);
        if (lane >= off) x += y;
      }
      if (lane == 31) misc[32 + warp] = x;
      __syncthreads();
      int before = 0, tot = 0;
      for (int w2 = 0; w2 < nt / 32; ++w2) {
        if (w2 < warp) before += misc[32 + w2];
        tot += misc[32 + w2];
      }
      if (f) gst[carry + before + x - 1] = pos;
      carry += tot;
      __syncthreads();
    }
    if (tid == 0) misc[2] = carry;
    __syncthreads();
    for (int g = tid; g < carry; g += nt) gsz[g] = (g + 1 < carry ? gst[g + 1] : B) - gst[g];
  }
  __syncthreads();
  // units. Beams with the same parent have the same chain, and their outputs must not depend on
  // how the beams are cut into units: a unit holds whole sibling groups of at most kUnitPos
  // positions while its distinct records stay <= up.maxAnc (greedy, left to right); a larger
  // group is cut into chunks of kUnitPos positions, each a unit of its own, so that every chunk
  // lists the chain's records in the same order (record u = chain slot u). A unit starting at
  // group g takes n_anc records for its first group and popc(fnew) new ones for each further
  // group, so its end is found by binary search on prefix sums of the group sizes and of the
  // new-record counts; one thread then follows the chain of unit starts.
  {
    const int ng = misc[2];
    int carry_s = 0, carry_c = 0;
    for (int base = 0; base < ng; base += nt) {
      const int g = base + tid;
      const int s1 = g < ng ? gsz[g] : 0;
      const int c1 = g < ng ? __popc(fnew[gst[g]]) : 0;
      int xs = s1, xc = c1;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int ys = __shfl_up_sync(kFull, xs, off), yc = __shfl_up_sync(kFull, xc, off);
        if (lane >= off) {
          xs += ys;
          xc += yc;
        }
      }
      if (lane == 31) {
        misc[32 + warp] = xs;
        misc[64 + warp] = xc;
      }
      __syncthreads();
      int bs = 0, bc = 0, ts = 0, tcn = 0;
      for (int w2 = 0; w2 < nt / 32; ++w2) {
        if (w2 < warp) {
          bs += misc[32 + w2];
          bc += misc[64 + w2];
        }
        ts += misc[32 + w2];
        tcn += misc[64 + w2];
      }
      if (g < ng) {
        PS[g + 1] = carry_s + bs + xs;
        PC[g + 1] = carry_c + bc + xc;
      }
      carry_s += ts;
      carry_c += tcn;
      __syncthreads();
    }
    if (tid == 0) {
      PS[0] = 0;
      PC[0] = 0;
    }
    __syncthreads();
    for (int g = tid; g < ng; g += nt) {
      // smallest j in (g, ng] at which adding group j breaks a limit (a group larger than
      // kUnitPos breaks the size limit by itself)
      int lo = g + 1, hi = ng;
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        const bool viol = PS[mid + 1] - PS[g] > kUnitPos || n_anc + PC[mid + 1] - PC[g + 1] > up.maxAnc;
        if (viol) hi = mid;
        else lo = mid + 1;
      }
      gnext[g] = lo;
    }
    __syncthreads();
    if (tid == 0) {
      int g = 0, k = 0;
      while (g < ng) {
        const int gs0 = gst[g], sz0 = gsz[g];
        if (sz0 > kUnitPos) {
          for (int off = 0; off < sz0; off += kUnitPos) {
            ustart[k] = gs0 + off;
            un[k] = min(kUnitPos, sz0 - off);
            uU[k] = n_anc;
            ++k;
          }
          ++g;
          continue;
        }
        const int j = gnext[g];
        ustart[k] = gs0;
        un[k] = PS[j] - PS[g];
        uU[k] = n_anc + PC[j] - PC[g + 1];
        ++k;
        g = j;
      }
      misc[0] = k;
    }
    __syncthreads();
    const int nu0 = misc[0];
    for (int x = tid; x < nu0 * kUnitPos; x += nt) {
      const int k = x / kUnitPos, j = x % kUnitPos;
      if (j < un[k]) uop[ustart[k] + j] = k;
    }
  }
  __syncthreads();
  const int nu = misc[0];
  int* rec_r = up.urec + size_t(r) * up.maxU * kUnitRecInts;
  // distinct records per (unit, slot): a warp per (unit, slot), a lane per position; the
  // record of position j is new if j is the unit's first position or the slot changed there
  const int nwarp = nt / 32;
  const unsigned lt = (1u << lane) - 1u;
  for (int x = warp; x < nu * n_anc; x += nwarp) {
    const int k = x / n_anc, s = x % n_anc;
    const bool in = lane < un[k];
    const bool f = in && (lane == 0 || ((fnew[ustart[k] + lane] >> s) & 1));
    const unsigned m = __ballot_sync(kFull, f);
    if (lane == 0) sdist[k * TA + s] = __popc(m);
  }
  __syncthreads();
  for (int k = tid; k < nu; k += nt) {              // counts -> offsets of each slot's records
    int run = 0;
    for (int s = 0; s < n_anc; ++s) {
      const int c = sdist[k * TA + s];
      sdist[k * TA + s] = run;
      run += c;
    }
  }
  __syncthreads();
  for (int x = warp; x < nu * n_anc; x += nwarp) {  // record list and per-position indices
    const int k = x / n_anc, s = x % n_anc;
    const int base = sdist[k * TA + s];
    const bool in = lane < un[k];
    const int pos = ustart[k] + lane;
    const bool f = in && (lane == 0 || ((fnew[pos] >> s) & 1));
    const unsigned m = __ballot_sync(kFull, f);
    const int c = __popc(m & lt) + (f ? 1 : 0);      // records up to and including this position
    if (f) rec_r[size_t(k) * kUnitRecInts + 36 + base + c - 1] = (s << 16) | spch[pos * TA + s];
    if (in) upos_s[pos * 16 + s] = uint8_t(base + c - 1);
  }
  __syncthreads();
  {                                                 // per-position record indices, 16 B a row
    const uint4* src = reinterpret_cast<const uint4*>(upos_s);
    uint4* dst = reinterpret_cast<uint4*>(up.upos + size_t(r) * B * 16);
    for (int pos = tid; pos < B; pos += nt) dst[pos] = src[pos];
  }
  for (int k = tid; k < nu; k += nt) {
    int* rk = rec_r + size_t(k) * kUnitRecInts;
    rk[0] = ustart[k] | (un[k] << 16);
    rk[1] = n_anc > 0 ? uU[k] : 0;
  }
  for (int pos = tid; pos < B; pos += nt) {
    const int k = uop[pos];
    rec_r[size_t(k) * kUnitRecInts + 4 + (pos - ustart[k])] = sperm[pos];
  }
  // unit counts; the last CTA to finish writes the prefix sums and resets the counter
  if (tid == 0) {
    up.ucnt[r] = nu;
    __threadfence();
    const unsigned ticket = atomicAdd(up.counter, 1u);
    misc[1] = ticket == gridDim.x - 1;
  }
  __syncthreads();
  if (misc[1]) {
    __threadfence();
    int carry = 0;
    int* wsum = misc + 32;
    for (int base = 0; base < a.R; base += nt) {
      const int v = base + tid < a.R ? __ldcg(up.ucnt + base + tid) : 0;
      int x = v;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(kFull, x, off);
        if (lane >= off) x += y;
      }
      if (lane == 31) wsum[warp] = x;
      __syncthreads();
      int before = 0, total = 0;
      for (int w = 0; w < nt / 32; ++w) {
        if (w < warp) before += wsum[w];
        total += wsum[w];
      }
      if (base + tid < a.R) up.uoff[base + tid] = carry + before + x - v;
      carry += total;
      __syncthreads();
    }
    if (tid == 0) {
      up.uoff[a.R] = carry;
      *up.counter = 0u;
    }
  }
}

cudaError_t launch_plan_units(const StepArgs& a, const UnitPlan& up, cudaStream_t stream) {
  const size_t smem = plan_units_smem(a.B, a.T_max);
  // the attribute is a limit, set once per device to the largest a handle may need (handles
  // whose plan needs more than the device offers are refused at create)
  static std::atomic<uint64_t> configured{0};
  cudaError_t e = once_per_device(configured, [] {
    int dev = 0, optin = 0;
    cudaError_t x = cudaGetDevice(&dev);
    if (x == cudaSuccess)
      x = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (x == cudaSuccess)
      x = cudaFuncSetAttribute(plan_units_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               optin);
    return x;
  });
  if (e != cudaSuccess) return e;
  plan_units_kernel<<<a.R, 512, smem, stream>>>(a, up);
  return cudaGetLastError();
}

}  // namespace ola
