// Bandwidth-bound passes of the step:
//   momentum_norm : M <- mu M + (1 - mu) G, U (Nesterov or not; or the two
//                   ANVIL momenta), writes U as the bf16 hi/lo iterate in the
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

__global__ void __launch_bounds__(256) momentum_norm_kernel(const __grid_constant__ MomParams p) {
  __shared__ float red[8];
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
  float ss = 0.0f;
  if ((C & 7) == 0) {
    for (long long e = e0 + threadIdx.x * 8; e < e1; e += 256 * 8) {
      const int prow = static_cast<int>(e / Cp);
      const int pcol = static_cast<int>(e - static_cast<long long>(prow) * Cp);
      float u[8];
      if (prow < R && pcol < C) {
        const long long i = ubase + static_cast<long long>(prow) * C + pcol;
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
      *reinterpret_cast<uint4*>(hi + e) = make_uint4(h[0], h[1], h[2], h[3]);
      *reinterpret_cast<uint4*>(lo + e) = make_uint4(l[0], l[1], l[2], l[3]);
    }
  } else {
    for (long long e = e0 + threadIdx.x; e < e1; e += 256) {
      const int prow = static_cast<int>(e / Cp);
      const int pcol = static_cast<int>(e - static_cast<long long>(prow) * Cp);
      float u = 0.0f;
      if (prow < R && pcol < C) {
        const long long i = ubase + static_cast<long long>(prow) * C + pcol;
        const float g = load1(io.grad, io.grad_dtype, i);
        float m = 0.0f, ms = 0.0f;
        if (p.mode != kMomNone) m = io.mom[i];
        if (p.mode == kMomAnvil) ms = io.mom_slow[i];
        u = momentum_elem(p, g, m, ms);
        ss = fmaf(u, u, ss);
        if (p.mode != kMomNone) io.mom[i] = m;
        if (p.mode == kMomAnvil) io.mom_slow[i] = ms;
      }
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
__device__ __forceinline__ float update_elem(const UpdParams& p, const UpdBank& io, float th,
                                             float o, float ms) {
  return param_update(p.mode, th, o, ms, io.step_scale, p.lr_wd);
}

__global__ void __launch_bounds__(256) update_kernel(const __grid_constant__ UpdParams p) {
  const long long tid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long nthr = static_cast<long long>(gridDim.x) * blockDim.x;
  for (int b = 0; b < p.nbanks; ++b) {
    const BankPlan& bp = p.bank[b];
    const UpdBank& io = p.io[b];
    if (!io.param) continue;  // updated by the last Newton-Schulz step
    const long long per = static_cast<long long>(bp.R) * bp.C;
    const long long n = per * bp.count;
    const __nv_bfloat16* hi = bp.hi[p.final_buf];
    const __nv_bfloat16* lo = bp.lo;
    const long long padded = static_cast<long long>(bp.Rp) * bp.Cp;
    const unsigned long long ngroups = static_cast<unsigned long long>(n / 8);
    if ((bp.C & 7) == 0 && ngroups < (1ull << 32)) {
      // groups of 8 consecutive elements of a row; 32-bit index arithmetic and
      // two independent groups per thread per pass (all loads issued first)
      const uint32_t ng = static_cast<uint32_t>(ngroups);
      const uint32_t gpr = static_cast<uint32_t>(bp.C / 8);
      const uint32_t R = static_cast<uint32_t>(bp.R);
      const uint32_t t32 = static_cast<uint32_t>(tid), n32 = static_cast<uint32_t>(nthr);
      for (uint32_t g0 = t32; g0 < ng; g0 += 2 * n32) {
        long long e[2], off[2];
        bool has[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const uint32_t g = g0 + static_cast<uint32_t>(u) * n32;
          has[u] = g < ng;
          const uint32_t gg = has[u] ? g : g0;
          const uint32_t row = gg / gpr;
          const uint32_t col = (gg - row * gpr) * 8u;
          const uint32_t mat = row / R;
          const uint32_t r = row - mat * R;
          e[u] = static_cast<long long>(gg) * 8;
          off[u] = (static_cast<long long>(mat) * bp.Rp + r) * bp.Cp + col;
        }
        float o[2][8], th[2][8], ms[2][8];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          if (!has[u]) continue;
          load8(hi, MUON_BF16, off[u], o[u]);
          if (p.mode != kUpdWriteO) load8(io.param, io.param_dtype, e[u], th[u]);
          if (p.mode == kUpdCautious) load8(io.mom_slow, MUON_F32, e[u], ms[u]);
          if (p.use_lo) {
            float l8[8];
            load8(lo, MUON_BF16, off[u], l8);
#pragma unroll
            for (int t = 0; t < 8; ++t) o[u][t] += l8[t];
          }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          if (!has[u]) continue;
          if (p.mode == kUpdWriteO) {
            store8(io.param, io.param_dtype, e[u], o[u]);
            continue;
          }
#pragma unroll
          for (int t = 0; t < 8; ++t)
            th[u][t] = stored(io.param_dtype,
                              update_elem(p, io, th[u][t], o[u][t], p.mode == kUpdCautious ? ms[u][t] : 0.0f));
          store8(io.param, io.param_dtype, e[u], th[u]);
          if (io.ema) {
            float em[8];
            load8(io.ema, MUON_F32, e[u], em);
#pragma unroll
            for (int t = 0; t < 8; ++t) em[t] = ema_elem(p.ema_beta, em[t], th[u][t]);
            store8(io.ema, MUON_F32, e[u], em);
          }
        }
      }
    } else if ((bp.C & 7) == 0) {
      for (long long g = tid; g < n / 8; g += nthr) {  // banks beyond 2^35 elements
        const long long e = g * 8;
        const long long mat = e / per;
        const long long rem = e - mat * per;
        const long long row = rem / bp.C;
        const long long off = mat * padded + row * bp.Cp + (rem - row * bp.C);
        float o[8], th[8], ms[8];
        load8(hi, MUON_BF16, off, o);
        if (p.use_lo) {
          float l8[8];
          load8(lo, MUON_BF16, off, l8);
#pragma unroll
          for (int t = 0; t < 8; ++t) o[t] += l8[t];
        }
        if (p.mode == kUpdWriteO) {
          store8(io.param, io.param_dtype, e, o);
          continue;
        }
        load8(io.param, io.param_dtype, e, th);
        if (p.mode == kUpdCautious) load8(io.mom_slow, MUON_F32, e, ms);
#pragma unroll
        for (int t = 0; t < 8; ++t)
          th[t] = stored(io.param_dtype, update_elem(p, io, th[t], o[t], p.mode == kUpdCautious ? ms[t] : 0.0f));
        store8(io.param, io.param_dtype, e, th);
        if (io.ema) {
          float em[8];
          load8(io.ema, MUON_F32, e, em);
#pragma unroll
          for (int t = 0; t < 8; ++t) em[t] = ema_elem(p.ema_beta, em[t], th[t]);
          store8(io.ema, MUON_F32, e, em);
        }
      }
    } else {
      for (long long e = tid; e < n; e += nthr) {
        const long long mat = e / per;
        const long long rem = e - mat * per;
        const long long row = rem / bp.C;
        const long long col = rem - row * bp.C;
        const long long off = mat * padded + row * bp.Cp + col;
        const float o = __bfloat162float(hi[off]) + (p.use_lo ? __bfloat162float(lo[off]) : 0.0f);
        if (p.mode == kUpdWriteO) {
          round_store1(io.param, io.param_dtype, e, o);
          continue;
        }
        const float th = load1(io.param, io.param_dtype, e);
        const float ms = p.mode == kUpdCautious ? io.mom_slow[e] : 0.0f;
        const float tn = round_store1(io.param, io.param_dtype, e, update_elem(p, io, th, o, ms));
        if (io.ema) io.ema[e] = ema_elem(p.ema_beta, io.ema[e], tn);
      }
    }
  }
}

cudaError_t launch_update(const UpdParams& p, long long total_elems, int num_sms, cudaStream_t s) {
  long long want = (total_elems / 16 + 255) / 256;  // two groups of 8 per thread per pass
  int grid = static_cast<int>(want < 1 ? 1 : (want > 8LL * num_sms ? 8LL * num_sms : want));
  update_kernel<<<grid, 256, 0, s>>>(p);
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
