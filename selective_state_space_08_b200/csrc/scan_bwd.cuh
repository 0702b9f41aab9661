// scan_bwd.cuh -- gradients of the Mamba-1 selective scan (sm_100a).
//
// For a loss with gradient dy with respect to y, with s_t = sum_n C[t,n]
// h[t,n] + D u_t, y_t = s_t silu(z_t) and h[t,n] = dA[t,n] h[t-1,n] +
// dt'_t B[t,n] u_t, the adjoint of the recurrence is
//   lambda[t,n] = ds_t C[t,n] + dA[t+1,n] lambda[t+1,n],  ds_t = dy_t silu(z_t),
// and every input receives its chain-rule terms through dt'_t, dA[t,n] =
// exp(dt'_t A[n]) and dt'_t B[t,n] u_t.  Page "从硬件感知到算法革命" section 1
// ("recomputation"): the states are rebuilt in the backward pass rather than
// stored by the forward one.
//
// Work decomposition.  One block per (batch, 32 channels), 16 warps: warp n
// owns state n of the block's 32 channels (lane c = channel d0 + c), so the
// sums over channels that B and C gradients need are warp reductions, and
// every thread keeps one state, one adjoint and one A entry in registers.
//  1. A forward sweep recomputes the states and stores a checkpoint (the
//     state before each 16-step block) in the workspace.
//  2. A reverse sweep takes the 16-step blocks from the last to the first:
//     it recomputes the block's states from its checkpoint into registers,
//     then runs the adjoint backwards through them.  dB and dC are summed
//     over the warp's channels and stored, one partial per block of
//     channels, in the workspace (a second kernel adds the partials: no
//     contended atomics on the shared B / C gradients);
//     the sums over states that du, ddelta and dz need go through shared
//     memory once per block of 16 steps; dA, dD and the bias gradient are
//     accumulated in registers and added atomically at the end.
// Data movement: 64-step tiles of u, delta, z, dy, B and C are staged into
// shared memory with loads coalesced along the steps, and dt', dt' u and
// ds = dy silu(z) are computed there once per element; the per-state sweeps
// read them from shared memory (rows padded to an odd number of words, so a
// warp's column reads hit 32 banks).
#pragma once
#include "common.cuh"

namespace ssm {

struct BwdParams {
  int64_t batch, dim, dstate, seqlen;
  const void* u;
  const void* delta;
  const void* z;
  const void* B;
  const void* C;
  const float* A;
  const float* D;
  const float* bias;
  int softplus;
  const float* h0;
  const float* dy;  // (batch, dim, seqlen) fp32
  // gradients, fp32; dA, dB, dC, dD, dbias are accumulated (zeroed by the host)
  float *du, *ddelta, *dz, *dA, *dB, *dC, *dD, *dbias, *dh0;
  float* ckpt;  // (batch, dim, 16, nblk): state before each 16-step block
  int64_t nblk;
  float* part;  // (2, channel blocks, batch, dstate, seqlen): per-block dB / dC sums
  int64_t nchb;  // channel blocks
};

namespace bwd {

constexpr int kCh = 32;       // channels per block (lanes)
constexpr int kStates = 16;   // warps: one state each
constexpr int kThreads = kCh * kStates;
constexpr int kBlk = 16;      // steps per recomputation block
static_assert(kBlk == kStates, "warp n finishes step n of each block");

constexpr int kTile = 64;     // steps staged in shared memory at a time
constexpr int kPadF = kTile + 1;  // fp32 rows of 65 words: column reads hit 32 banks
template <typename T>
struct RawRow {  // elements per staged row: an odd number of 32-bit words
  static constexpr int kLen = sizeof(T) == 2 ? kTile + 2 : kTile + 1;
};

template <typename T>
struct Smem {
  // the tile's inputs, [row][step]
  T u[kCh][RawRow<T>::kLen];
  T dl[kCh][RawRow<T>::kLen];
  T z[kCh][RawRow<T>::kLen];
  float dy[kCh][kPadF];
  T Bm[kStates][RawRow<T>::kLen];
  T Cm[kStates][RawRow<T>::kLen];
  // per element, once per channel: dt', dt' u, ds = dy silu(z)
  float dtp[kCh][kPadF];
  float dtu[kCh][kPadF];
  float ds[kCh][kPadF];
  // partial sums over states of one 16-step block, per (state, step, channel)
  float part_du[kStates][kBlk][kCh];
  float part_dt[kStates][kBlk][kCh];
  float part_s[kStates][kBlk][kCh];
  float red_dD[kBlk][kCh];  // per (step slot, channel): running dD / bias sums
  float red_db[kBlk][kCh];
};

__device__ __forceinline__ float softplus_grad_f(float s) {
  return s > 20.f ? 1.f : 1.f / (1.f + __expf(-s));
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <typename T>
__global__ void __launch_bounds__(kThreads) scan_bwd_kernel(const BwdParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Smem<T>& sm = *reinterpret_cast<Smem<T>*>(smem_raw);
  const int tid = threadIdx.x;
  const int c = tid % kCh;   // channel within the block
  const int n = tid / kCh;   // state (warp)
  const int64_t b = blockIdx.y;
  const int64_t d0 = static_cast<int64_t>(blockIdx.x) * kCh;
  const int64_t d = d0 + c;
  const int N = static_cast<int>(p.dstate);
  const int64_t L = p.seqlen;
  const bool ch_ok = d < p.dim;
  const bool ok = ch_ok && n < N;  // this thread owns a real state
  const int64_t row = b * p.dim + d;
  const T* gu = static_cast<const T*>(p.u);
  const T* gdl = static_cast<const T*>(p.delta);
  const T* gz = static_cast<const T*>(p.z);
  const T* gB = static_cast<const T*>(p.B);
  const T* gC = static_cast<const T*>(p.C);
  const float An = ok ? p.A[d * N + n] : 0.f;
  const float Dd = (ch_ok && p.D) ? p.D[d] : 0.f;
  const float bias = (ch_ok && p.bias) ? p.bias[d] : 0.f;
  const int nchv = static_cast<int>(imin64(kCh, p.dim - d0));  // valid channels of the block
  const int64_t ntile = (L + kTile - 1) / kTile;

  // Stage steps [t0, t0 + len) of the block's rows (coalesced along the
  // steps; zero past the end, past the last channel and past the last state),
  // then compute dt', dt' u and (reverse sweep) ds once per element.
  auto stage = [&](int64_t t0, int len, bool rev) {
    for (int i = tid; i < kCh * kTile; i += kThreads) {
      const int r = i / kTile, e = i % kTile;
      const bool v = r < nchv && e < len;
      const int64_t g = (b * p.dim + d0 + r) * L + t0 + e;
      sm.u[r][e] = v ? gu[g] : from_f32<T>(0.f);
      sm.dl[r][e] = v ? gdl[g] : from_f32<T>(0.f);
      if (rev) {
        sm.z[r][e] = (v && gz != nullptr) ? gz[g] : from_f32<T>(0.f);
        sm.dy[r][e] = v ? p.dy[g] : 0.f;
      }
    }
    for (int i = tid; i < kStates * kTile; i += kThreads) {
      const int r = i / kTile, e = i % kTile;
      const bool v = r < N && e < len;
      const int64_t g = (b * N + r) * L + t0 + e;
      sm.Bm[r][e] = v ? gB[g] : from_f32<T>(0.f);
      if (rev) sm.Cm[r][e] = v ? gC[g] : from_f32<T>(0.f);
    }
    __syncthreads();
    for (int i = tid; i < kCh * kTile; i += kThreads) {
      const int r = i / kTile, e = i % kTile;
      float dt = 0.f;
      if (r < nchv && e < len) {
        const float sarg = to_f32<T>(sm.dl[r][e]) + (p.bias ? p.bias[d0 + r] : 0.f);
        dt = p.softplus ? softplus_f(sarg) : sarg;
      }
      sm.dtp[r][e] = dt;
      sm.dtu[r][e] = dt * to_f32<T>(sm.u[r][e]);
      if (rev) {
        const float gate = gz != nullptr ? silu_f(to_f32<T>(sm.z[r][e])) : 1.f;
        sm.ds[r][e] = sm.dy[r][e] * gate;
      }
    }
    __syncthreads();
  };

  // ---- 1. forward sweep: checkpoints (state before each 16-step block) ----------------
  float h = (ok && p.h0) ? p.h0[row * N + n] : 0.f;
  for (int64_t k = 0; k < ntile; ++k) {
    const int64_t t0 = k * kTile;
    const int len = static_cast<int>(imin64(kTile, L - t0));
    stage(t0, len, false);
    for (int q = 0; q * kBlk < len; ++q) {
      if (ok) p.ckpt[(row * kStates + n) * p.nblk + k * (kTile / kBlk) + q] = h;
      const int e1 = min(len, (q + 1) * kBlk);
#pragma unroll 4
      for (int e = q * kBlk; e < e1; ++e)
        h = fmaf(__expf(sm.dtp[c][e] * An), h, sm.dtu[c][e] * to_f32<T>(sm.Bm[n < N ? n : 0][e]) *
                                                       (n < N ? 1.f : 0.f));
    }
    __syncthreads();  // the next tile is staged over this one
  }

  // ---- 2. reverse sweep ------------------------------------------------------------------
  float lam = 0.f, dA_acc = 0.f;
  float dD_acc = 0.f, db_acc = 0.f;  // this thread's (step slot n, channel c) share
  for (int64_t k = ntile - 1; k >= 0; --k) {
    const int64_t tk = k * kTile;
    const int len = static_cast<int>(imin64(kTile, L - tk));
    stage(tk, len, true);
    for (int q = (len - 1) / kBlk; q >= 0; --q) {
      const int e0 = q * kBlk;                 // block start within the tile
      const int nt = min(kBlk, len - e0);      // steps of the block
      const int64_t t0 = tk + e0;
      const int nr = n < N ? n : 0;            // a valid row of B / C for every warp
      const float on = n < N ? 1.f : 0.f;
      // recompute the block's states: hs[i] = h[t0 + i], hp[i] = h[t0 + i - 1]
      float hs[kBlk], hp[kBlk], dts[kBlk], as[kBlk];
      float hv = ok ? p.ckpt[(row * kStates + n) * p.nblk + k * (kTile / kBlk) + q] : 0.f;
#pragma unroll
      for (int i = 0; i < kBlk; ++i) {
        float dt = 0.f, a = 1.f, inc = 0.f;
        if (i < nt) {
          dt = sm.dtp[c][e0 + i];
          a = __expf(dt * An);
          inc = sm.dtu[c][e0 + i] * to_f32<T>(sm.Bm[nr][e0 + i]) * on;
        }
        hp[i] = hv;
        hv = fmaf(a, hv, inc);
        hs[i] = hv;
        dts[i] = dt;
        as[i] = a;
      }
      // adjoint, backwards through the block
#pragma unroll
      for (int i = kBlk - 1; i >= 0; --i) {
        float pdu = 0.f, pdt = 0.f, ps = 0.f;
        if (i < nt) {
          const int e = e0 + i;
          const int64_t t = t0 + i;
          const float uv = to_f32<T>(sm.u[c][e]);
          const float Bv = to_f32<T>(sm.Bm[nr][e]) * on, Cv = to_f32<T>(sm.Cm[nr][e]) * on;
          const float ds = sm.ds[c][e];
          lam = fmaf(ds, Cv, lam);
          const float gC = warp_sum(ds * hs[i]);
          const float gB = warp_sum(lam * sm.dtu[c][e]);
          if (c == 0 && n < N) {
            const int64_t slot = ((static_cast<int64_t>(blockIdx.x) * p.batch + b) * N + n) * L + t;
            p.part[slot] = gB;
            p.part[p.nchb * p.batch * N * L + slot] = gC;
          }
          pdu = lam * dts[i] * Bv;
          pdt = lam * (An * as[i] * hp[i] + Bv * uv);
          ps = Cv * hs[i];
          dA_acc = fmaf(lam * dts[i] * as[i], hp[i], dA_acc);
          lam *= as[i];
        }
        sm.part_du[n][i][c] = pdu;
        sm.part_dt[n][i][c] = pdt;
        sm.part_s[n][i][c] = ps;
      }
      __syncthreads();
      // thread (slot n, channel c) finishes step t0 + n of channel c
      {
        const int i = n;  // step within the block
        if (i < nt && ch_ok) {
          const int e = e0 + i;
          const int64_t t = t0 + i;
          float sdu = 0.f, sdt = 0.f, ss = 0.f;
#pragma unroll
          for (int kk = 0; kk < kStates; ++kk) {
            sdu += sm.part_du[kk][i][c];
            sdt += sm.part_dt[kk][i][c];
            ss += sm.part_s[kk][i][c];
          }
          const float uv = to_f32<T>(sm.u[c][e]);
          const float dyv = sm.dy[c][e];
          if (gz != nullptr) {
            const float zv = to_f32<T>(sm.z[c][e]);
            const float sg = 1.f / (1.f + __expf(-zv));
            if (p.dz) p.dz[row * L + t] = dyv * (ss + Dd * uv) * (sg * (1.f + zv * (1.f - sg)));
          }
          const float ds = sm.ds[c][e];
          if (p.du) p.du[row * L + t] = fmaf(ds, Dd, sdu);
          const float sarg = to_f32<T>(sm.dl[c][e]) + bias;
          const float ddt = p.softplus ? sdt * softplus_grad_f(sarg) : sdt;
          if (p.ddelta) p.ddelta[row * L + t] = ddt;
          dD_acc = fmaf(ds, uv, dD_acc);
          db_acc += ddt;
        }
      }
      __syncthreads();  // the partial sums are rewritten by the next block
    }
  }

  // ---- 3. parameter gradients -------------------------------------------------------------
  if (ok) {
    atomicAdd(&p.dA[d * N + n], dA_acc);
    if (p.dh0) p.dh0[row * N + n] = lam;
  }
  sm.red_dD[n][c] = dD_acc;
  sm.red_db[n][c] = db_acc;
  __syncthreads();
  if (n == 0 && ch_ok) {
    float sD = 0.f, sb = 0.f;
#pragma unroll
    for (int kk = 0; kk < kBlk; ++kk) {
      sD += sm.red_dD[kk][c];
      sb += sm.red_db[kk][c];
    }
    if (p.dD) atomicAdd(&p.dD[d], sD);
    if (p.dbias) atomicAdd(&p.dbias[d], sb);
  }
}

// dB and dC: the sum over channel blocks of the per-block partials; one
// thread per (batch, state, step), reads coalesced along the steps.
__global__ void scan_bwd_reduce_bc(const BwdParams p) {
  const int64_t per = p.batch * p.dstate * p.seqlen;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= per) return;
  float sb = 0.f, sc = 0.f;
  for (int64_t x = 0; x < p.nchb; ++x) {
    sb += p.part[x * per + i];
    sc += p.part[(p.nchb + x) * per + i];
  }
  p.dB[i] = sb;
  p.dC[i] = sc;
}

}  // namespace bwd
}  // namespace ssm
