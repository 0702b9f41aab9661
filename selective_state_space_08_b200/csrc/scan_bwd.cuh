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
// This kernel favours a direct, checkable structure over speed: every thread
// of a channel recomputes dt' and the gate, and the sequence loads of a warp
// touch 32 rows.
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

struct Smem {
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
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
  const int tid = threadIdx.x;
  const int c = tid % kCh;   // channel within the block
  const int n = tid / kCh;   // state
  const int64_t b = blockIdx.y;
  const int64_t d = static_cast<int64_t>(blockIdx.x) * kCh + c;
  const int N = static_cast<int>(p.dstate);
  const int64_t L = p.seqlen;
  const bool ch_ok = d < p.dim;
  const bool ok = ch_ok && n < N;  // this thread owns a real state
  const int64_t row = b * p.dim + d;
  const T* u = static_cast<const T*>(p.u);
  const T* dl = static_cast<const T*>(p.delta);
  const T* zt = static_cast<const T*>(p.z);
  const T* Bm = static_cast<const T*>(p.B);
  const T* Cm = static_cast<const T*>(p.C);
  const float An = ok ? p.A[d * N + n] : 0.f;
  const float Dd = (ch_ok && p.D) ? p.D[d] : 0.f;
  const float bias = (ch_ok && p.bias) ? p.bias[d] : 0.f;

  auto in = [&](const T* base, int64_t t) { return ch_ok ? to_f32<T>(base[row * L + t]) : 0.f; };
  auto bc = [&](const T* base, int64_t t) {
    return ok ? to_f32<T>(base[(b * N + n) * L + t]) : 0.f;
  };
  auto step_size = [&](int64_t t) {
    const float s = in(dl, t) + bias;
    return p.softplus ? softplus_f(s) : s;
  };

  // ---- 1. forward sweep: checkpoints -----------------------------------------------
  float h = (ok && p.h0) ? p.h0[row * N + n] : 0.f;
  for (int64_t j = 0; j < p.nblk; ++j) {
    if (ok) p.ckpt[(row * kStates + n) * p.nblk + j] = h;
    const int64_t t1 = imin64(L, (j + 1) * kBlk);
    for (int64_t t = j * kBlk; t < t1; ++t) {
      const float dt = step_size(t);
      h = fmaf(__expf(dt * An), h, dt * bc(Bm, t) * in(u, t));
    }
  }

  // ---- 2. reverse sweep ------------------------------------------------------------------
  float lam = 0.f, dA_acc = 0.f;
  float dD_acc = 0.f, db_acc = 0.f;  // this thread's (step slot n, channel c) share
  for (int64_t j = p.nblk - 1; j >= 0; --j) {
    const int64_t t0 = j * kBlk;
    const int nt = static_cast<int>(imin64(kBlk, L - t0));
    // recompute the block's states: hs[i] = h[t0 + i], hp[i] = h[t0 + i - 1]
    float hs[kBlk], hp[kBlk], dts[kBlk], as[kBlk];
    float hv = ok ? p.ckpt[(row * kStates + n) * p.nblk + j] : 0.f;
#pragma unroll
    for (int i = 0; i < kBlk; ++i) {
      float dt = 0.f, a = 1.f, inc = 0.f;
      if (i < nt) {
        dt = step_size(t0 + i);
        a = __expf(dt * An);
        inc = dt * bc(Bm, t0 + i) * in(u, t0 + i);
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
        const int64_t t = t0 + i;
        const float uv = in(u, t), Bv = bc(Bm, t), Cv = bc(Cm, t);
        float gate = 1.f;
        if (zt != nullptr) gate = silu_f(in(zt, t));
        const float ds = (ch_ok ? p.dy[row * L + t] : 0.f) * gate;
        lam = fmaf(ds, Cv, lam);
        const float gC = warp_sum(ds * hs[i]);
        const float gB = warp_sum(lam * dts[i] * uv);
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
        const int64_t t = t0 + i;
        float sdu = 0.f, sdt = 0.f, ss = 0.f;
#pragma unroll
        for (int k = 0; k < kStates; ++k) {
          sdu += sm.part_du[k][i][c];
          sdt += sm.part_dt[k][i][c];
          ss += sm.part_s[k][i][c];
        }
        const float uv = in(u, t);
        const float dyv = p.dy[row * L + t];
        float gate = 1.f;
        if (zt != nullptr) {
          const float zv = in(zt, t);
          const float sg = 1.f / (1.f + __expf(-zv));
          gate = zv * sg;
          if (p.dz) p.dz[row * L + t] = dyv * (ss + Dd * uv) * (sg * (1.f + zv * (1.f - sg)));
        }
        const float ds = dyv * gate;
        if (p.du) p.du[row * L + t] = fmaf(ds, Dd, sdu);
        const float sarg = in(dl, t) + bias;
        const float ddt = p.softplus ? sdt * softplus_grad_f(sarg) : sdt;
        if (p.ddelta) p.ddelta[row * L + t] = ddt;
        dD_acc = fmaf(ds, uv, dD_acc);
        db_acc += ddt;
      }
    }
    __syncthreads();  // the partial sums are rewritten by the next block
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
    for (int k = 0; k < kBlk; ++k) {
      sD += sm.red_dD[k][c];
      sb += sm.red_db[k][c];
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
