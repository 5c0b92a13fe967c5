// Bandwidth-bound passes of the step:
//   momentum_norm : M <- mu M + (1 - mu) G (or the SGD form M <- mu M + G),
//                   U (Nesterov or not; or the two ANVIL momenta), writes U as
//                   the bf16 hi/lo iterate in the
//                   padded working layout and per-block partial sums of U^2
//   norm_finalize : 1 / (||U||_F + eps) per matrix from the partials, in a
//                   fixed order (deterministic); resets the matrix's
//                   Newton-Schulz completion counters
//   update        : theta <- theta (1 - lr wd [mask]) - lr s O, optional EMA
//   ema / blend   : standalone EMA and readout blend
// ("Muonとは": momentum as a moving average of the gradient; "ANVIL II와 가중치
// 평균": two momenta, cautious decay, the EMA equation and the 35/65 blend.)
// Vector path: 8 consecutive elements per thread (16-byte bf16 / 2 x 16-byte
// fp32 accesses) when the row length is a multiple of 8; scalar path otherwise.
#include <cuda_runtime.h>

#include "plan.cuh"
#include "ptx.cuh"

namespace muon {

__device__ __forceinline__ void load8(const void* base, int dtype, long long i, float (&x)[8]) {
  if (dtype == MUON_BF16) {
    const uint4 w = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(base) + i);
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      x[2 * h] = bf16_lo_f(ww[h]);
      x[2 * h + 1] = bf16_hi_f(ww[h]);
    }
  } else {
    const float4* f = reinterpret_cast<const float4*>(static_cast<const float*>(base) + i);
    const float4 a = f[0], b = f[1];
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  }
}

__device__ __forceinline__ void store8(void* base, int dtype, long long i, const float (&x)[8]) {
  if (dtype == MUON_BF16) {
    *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(base) + i) =
        make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                   pack_bf16x2(x[6], x[7]));
  } else {
    float4* f = reinterpret_cast<float4*>(static_cast<float*>(base) + i);
    f[0] = make_float4(x[0], x[1], x[2], x[3]);
    f[1] = make_float4(x[4], x[5], x[6], x[7]);
  }
}

__device__ __forceinline__ float load1(const void* base, int dtype, long long i) {
  if (dtype == MUON_BF16) return __bfloat162float(static_cast<const __nv_bfloat16*>(base)[i]);
  return static_cast<const float*>(base)[i];
}

__device__ __forceinline__ float round_store1(void* base, int dtype, long long i, float x) {
  if (dtype == MUON_BF16) {
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    static_cast<__nv_bfloat16*>(base)[i] = h;
    return __bfloat162float(h);
  }
  static_cast<float*>(base)[i] = x;
  return x;
}

// U for one element; updates the momentum values in place.
__device__ __forceinline__ float momentum_elem(const MomParams& p, float g, float& m, float& ms) {
  if (p.mode == kMomNone) return g;
  if (p.mode == kMomAnvil) {
    m = fmaf(p.mu, m, (1.0f - p.mu) * g);
    ms = fmaf(p.mu_slow, ms, (1.0f - p.mu_slow) * g);
    return m;
  }
  const float gw = p.sgd ? g : (1.0f - p.mu) * g;  // SGD form or moving average
  m = fmaf(p.mu, m, gw);
  return p.nesterov ? fmaf(p.mu, m, gw) : m;
}

__device__ __forceinline__ float block_sum_256(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float t = 0.0f;
  if (threadIdx.x == 0) {
    for (int w = 0; w < 8; ++w) t += red[w];
  }
  return t;
}

// Every pass that writes the caller's buffers first reads the workspace's
// status word: while it holds an error (a bounded wait of an earlier launch
// ran out; the word is sticky until the caller clears it) the pass writes
// nothing, so a failed step leaves params, EMA and O as they were, and later
// steps leave the momenta too.
__device__ __forceinline__ bool status_clear(const int* status) {
  return status == nullptr || *reinterpret_cast<const volatile int*>(status) == 0;
}

__global__ void __launch_bounds__(256) momentum_norm_kernel(const __grid_constant__ MomParams p) {
  __shared__ float red[8];
  if (!status_clear(p.status)) return;
  const int blk = blockIdx.x;
  int b = 0;
  while (b + 1 < p.nbanks && blk >= p.block_begin[b + 1]) ++b;
  const BankPlan& bp = p.bank[b];
  const MomBank& io = p.io[b];
  const int local = blk - p.block_begin[b];
  const int mat = local / bp.chunks;
  const int chunk = local - mat * bp.chunks;
  const long long padded = static_cast<long long>(bp.Rp) * bp.Cp;
  const long long e0 = static_cast<long long>(chunk) * kChunk;
  const long long e1 = min(e0 + kChunk, padded);
  __nv_bfloat16* hi = bp.hi[0] + mat * padded;
  __nv_bfloat16* lo = bp.lo + mat * padded;
  const long long ubase = static_cast<long long>(mat) * bp.R * bp.C;
  const int R = bp.R, C = bp.C, Cp = bp.Cp;
  // buffer extents for the debug build's checks: logical and padded elements
  const long long nlog = static_cast<long long>(bp.count) * R * C;
  const long long nwork = static_cast<long long>(bp.count) * padded;
  const long long wbase = static_cast<long long>(mat) * padded;
  float ss = 0.0f;
  if ((C & 7) == 0) {
    for (long long e = e0 + threadIdx.x * 8; e < e1; e += 256 * 8) {
      const int prow = static_cast<int>(e / Cp);
      const int pcol = static_cast<int>(e - static_cast<long long>(prow) * Cp);
      const long long i = ubase + static_cast<long long>(prow) * C + pcol;
      float u[8];
      if (prow < R && pcol < C && in_bounds(i + 8 <= nlog, p.status)) {
        float g[8], m[8], ms[8];
        load8(io.grad, io.grad_dtype, i, g);
        if (p.mode != kMomNone) load8(io.mom, MUON_F32, i, m);
        if (p.mode == kMomAnvil) load8(io.mom_slow, MUON_F32, i, ms);
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          u[t] = momentum_elem(p, g[t], m[t], ms[t]);
          ss = fmaf(u[t], u[t], ss);
        }
        if (p.mode != kMomNone) store8(io.mom, MUON_F32, i, m);
        if (p.mode == kMomAnvil) store8(io.mom_slow, MUON_F32, i, ms);
      } else {
#pragma unroll
        for (int t = 0; t < 8; ++t) u[t] = 0.0f;
      }
      uint32_t h[4], l[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        h[q] = pack_bf16x2(u[2 * q], u[2 * q + 1]);
        l[q] = pack_bf16x2(u[2 * q] - bf16_lo_f(h[q]), u[2 * q + 1] - bf16_hi_f(h[q]));
      }
      if (!in_bounds(wbase + e + 8 <= nwork, p.status)) continue;
      *reinterpret_cast<uint4*>(hi + e) = make_uint4(h[0], h[1], h[2], h[3]);
      *reinterpret_cast<uint4*>(lo + e) = make_uint4(l[0], l[1], l[2], l[3]);
    }
  } else {
    for (long long e = e0 + threadIdx.x; e < e1; e += 256) {
      const int prow = static_cast<int>(e / Cp);
      const int pcol = static_cast<int>(e - static_cast<long long>(prow) * Cp);
      const long long i = ubase + static_cast<long long>(prow) * C + pcol;
      float u = 0.0f;
      if (prow < R && pcol < C && in_bounds(i < nlog, p.status)) {
        const float g = load1(io.grad, io.grad_dtype, i);
        float m = 0.0f, ms = 0.0f;
        if (p.mode != kMomNone) m = io.mom[i];
        if (p.mode == kMomAnvil) ms = io.mom_slow[i];
        u = momentum_elem(p, g, m, ms);
        ss = fmaf(u, u, ss);
        if (p.mode != kMomNone) io.mom[i] = m;
        if (p.mode == kMomAnvil) io.mom_slow[i] = ms;
      }
      if (!in_bounds(wbase + e < nwork, p.status)) continue;
      const __nv_bfloat16 h = __float2bfloat16_rn(u);
      hi[e] = h;
      lo[e] = __float2bfloat16_rn(u - __bfloat162float(h));
    }
  }
  const float tot = block_sum_256(ss, red);
  if (threadIdx.x == 0) bp.partial[static_cast<long long>(mat) * bp.chunks + chunk] = tot;
}

// One warp per matrix: fixed-order sum of the partials in double.
__global__ void __launch_bounds__(128) norm_finalize_kernel(const __grid_constant__ MomParams p,
                                                            int total_mats) {
  const int gm = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (gm >= total_mats) return;
  int b = 0;
  while (b + 1 < p.nbanks && gm >= p.mat_begin[b + 1]) ++b;
  const BankPlan& bp = p.bank[b];
  const int mat = gm - p.mat_begin[b];
  const float* part = bp.partial + static_cast<long long>(mat) * bp.chunks;
  double s = 0.0;
  for (int i = lane; i < bp.chunks; i += 32) s += static_cast<double>(part[i]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) bp.scale[mat] = static_cast<float>(1.0 / (sqrt(s) + static_cast<double>(p.eps)));
  // the Newton-Schulz chain's per-matrix completion counters start at zero
  if (lane < 4) bp.counters[4 * mat + lane] = 0;
}

cudaError_t launch_momentum_norm(const MomParams& p, int total_blocks, int total_mats,
                                 cudaStream_t s) {
  momentum_norm_kernel<<<total_blocks, 256, 0, s>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  norm_finalize_kernel<<<(total_mats + 3) / 4, 128, 0, s>>>(p, total_mats);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ update
// One block per (matrix, kChunk padded elements), the momentum pass's grid;
// each thread takes one group of 8 at a time, so few registers and a full
// SM of resident blocks keep enough loads in flight for HBM (a grid-stride
// version with two groups per thread reached about half of the bandwidth).
template <int Mode>
__global__ void __launch_bounds__(256) update_kernel(const __grid_constant__ UpdParams p) {
  if (!status_clear(p.status)) return;  // the chain did not finish: O is not valid
  const int blk = blockIdx.x;
  int b = 0;
  while (b + 1 < p.nbanks && blk >= p.block_begin[b + 1]) ++b;
  const BankPlan& bp = p.bank[b];
  const UpdBank& io = p.io[b];
  const int local = blk - p.block_begin[b];
  const int mat = local / bp.chunks;
  const int chunk = local - mat * bp.chunks;
  const long long padded = static_cast<long long>(bp.Rp) * bp.Cp;
  const long long e0 = static_cast<long long>(chunk) * kChunk;
  const long long e1 = min(e0 + kChunk, padded);
  const __nv_bfloat16* hi = bp.hi[p.final_buf] + mat * padded;
  const __nv_bfloat16* lo = bp.lo + mat * padded;
  const long long ubase = static_cast<long long>(mat) * bp.R * bp.C;
  const int R = bp.R, C = bp.C, Cp = bp.Cp;
  const long long nlog = static_cast<long long>(bp.count) * R * C;  // debug-build extents
  const long long nwork = static_cast<long long>(bp.count) * padded;
  const long long wbase = static_cast<long long>(mat) * padded;
  if ((C & 7) == 0) {
    for (long long e = e0 + threadIdx.x * 8; e < e1; e += 256 * 8) {
      const int prow = static_cast<int>(e / Cp);
      const int pcol = static_cast<int>(e - static_cast<long long>(prow) * Cp);
      if (prow >= R || pcol >= C) continue;
      const long long i = ubase + static_cast<long long>(prow) * C + pcol;
      if (!in_bounds(i + 8 <= nlog && wbase + e + 8 <= nwork, p.status)) continue;
      float o[8], th[8], ms[8];
      load8(hi, MUON_BF16, e, o);
      if (p.use_lo) {
        float l8[8];
        load8(lo, MUON_BF16, e, l8);
#pragma unroll
        for (int t = 0; t < 8; ++t) o[t] += l8[t];
      }
      if (Mode == kUpdWriteO) {
        store8(io.param, io.param_dtype, i, o);
        continue;
      }
      load8(io.param, io.param_dtype, i, th);
      if (Mode == kUpdCautious) load8(io.mom_slow, MUON_F32, i, ms);
#pragma unroll
      for (int t = 0; t < 8; ++t)
        th[t] = stored(io.param_dtype, param_update(Mode, th[t], o[t], ms[t], io.step_scale, p.lr_wd));
      store8(io.param, io.param_dtype, i, th);
      if (io.ema) {
        float em[8];
        load8(io.ema, MUON_F32, i, em);
#pragma unroll
        for (int t = 0; t < 8; ++t) em[t] = ema_elem(p.ema_beta, em[t], th[t]);
        store8(io.ema, MUON_F32, i, em);
      }
    }
  } else {
    for (long long e = e0 + threadIdx.x; e < e1; e += 256) {
      const int prow = static_cast<int>(e / Cp);
      const int pcol = static_cast<int>(e - static_cast<long long>(prow) * Cp);
      if (prow >= R || pcol >= C) continue;
      const long long i = ubase + static_cast<long long>(prow) * C + pcol;
      if (!in_bounds(i < nlog && wbase + e < nwork, p.status)) continue;
      const float o = __bfloat162float(hi[e]) + (p.use_lo ? __bfloat162float(lo[e]) : 0.0f);
      if (Mode == kUpdWriteO) {
        round_store1(io.param, io.param_dtype, i, o);
        continue;
      }
      const float th = load1(io.param, io.param_dtype, i);
      const float ms = Mode == kUpdCautious ? io.mom_slow[i] : 0.0f;
      const float tn = round_store1(io.param, io.param_dtype, i, param_update(Mode, th, o, ms, io.step_scale, p.lr_wd));
      if (io.ema) io.ema[i] = ema_elem(p.ema_beta, io.ema[i], tn);
    }
  }
}

cudaError_t launch_update(const UpdParams& p, int total_blocks, cudaStream_t s) {
  if (p.mode == kUpdCautious)
    update_kernel<kUpdCautious><<<total_blocks, 256, 0, s>>>(p);
  else if (p.mode == kUpdWriteO)
    update_kernel<kUpdWriteO><<<total_blocks, 256, 0, s>>>(p);
  else
    update_kernel<kUpdDecoupled><<<total_blocks, 256, 0, s>>>(p);
  return cudaGetLastError();
}

// ---------------------------------------------------------- EMA and blend
__global__ void __launch_bounds__(256) ema_kernel(float* ema, const void* param, int dtype,
                                                  long long n, float beta) {
  const long long tid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long nthr = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = tid; i < n; i += nthr)
    ema[i] = ema_elem(beta, ema[i], load1(param, dtype, i));
}

__global__ void __launch_bounds__(256) blend_kernel(const void* theta, int tdtype, const float* ema,
                                                    void* out, int odtype, long long n, float w) {
  const long long tid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long nthr = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = tid; i < n; i += nthr)
    round_store1(out, odtype, i, fmaf(w, load1(theta, tdtype, i), (1.0f - w) * ema[i]));
}

static int grid_for(long long n, int num_sms) {
  long long want = (n + 255) / 256;
  if (want < 1) want = 1;
  if (want > 16LL * num_sms) want = 16LL * num_sms;
  return static_cast<int>(want);
}

cudaError_t launch_ema(float* ema, const void* param, int param_dtype, long long n, float beta,
                       int num_sms, cudaStream_t s) {
  ema_kernel<<<grid_for(n, num_sms), 256, 0, s>>>(ema, param, param_dtype, n, beta);
  return cudaGetLastError();
}

cudaError_t launch_blend(const void* theta, int theta_dtype, const float* ema, void* out,
                         int out_dtype, long long n, float w_final, int num_sms, cudaStream_t s) {
  blend_kernel<<<grid_for(n, num_sms), 256, 0, s>>>(theta, theta_dtype, ema, out, out_dtype, n,
                                                    w_final);
  return cudaGetLastError();
}

}  // namespace muon
