// C ABI of the library: argument validation, workspace planning, TMA tensor
// maps and the launch sequence of one optimizer step. Nothing here allocates
// or synchronises on the step path; all work is enqueued on the caller's stream.
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstring>
#include <mutex>
#include <utility>

#include "muon_b200.h"
#include "plan.cuh"
#include "tiles.cuh"

using namespace muon;

namespace {

// ------------------------------------------------------------ process state
struct DebugState {
  int fault = 0;
  double wait_limit_s = 2.0;
};
DebugState g_debug;

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
cudaEvent_t g_ev_before = nullptr, g_ev_after = nullptr;
std::mutex g_mu;

struct DeviceState {
  bool ready = false;
  int sms = 0;
  int max_pairs = 0;  // CTA pairs of the Newton-Schulz chain that fit on the device at once
};
DeviceState g_dev[64];

muon_status device_state(int* sms, int* max_pairs = nullptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MUON_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
      return MUON_ERR_CUDA;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  DeviceState& d = g_dev[dev];
  if (!d.ready) {
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return MUON_ERR_CUDA;
    if (ns_gemm_prepare(&d.max_pairs) != cudaSuccess) return MUON_ERR_CUDA;
    d.ready = true;
  }
  *sms = d.sms;
  if (max_pairs) *max_pairs = d.max_pairs;
  return MUON_OK;
}

// ------------------------------------------------------------ validation
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool dtype_ok(int32_t d) { return d == MUON_F32 || d == MUON_BF16; }
inline int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }
inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

constexpr size_t kHeaderBytes = 4096;  // device status word at offset 0

muon_status check_shape(int64_t count, int64_t rows, int64_t cols) {
  if (count < 1 || rows < 1 || cols < 1) return MUON_ERR_SHAPE;
  // bound each factor first so that the products below cannot overflow
  if (count >= (int64_t(1) << 31) || rows >= (int64_t(1) << 24) || cols >= (int64_t(1) << 24))
    return MUON_ERR_SHAPE;
  const int64_t Rp = round_up(rows, kPad), Cp = round_up(cols, kPad);
  const int64_t rp = rows > cols ? Cp : Rp;
  // TMA coordinates and tile indices are 32-bit
  if (count * Rp >= (int64_t(1) << 31) || count * rp >= (int64_t(1) << 31)) return MUON_ERR_SHAPE;
  if (Rp >= (int64_t(1) << 24) || Cp >= (int64_t(1) << 24)) return MUON_ERR_SHAPE;
  const int64_t tiles = count * (Rp / kTile) * (Cp / kTile);
  const int64_t chunks = (Rp * Cp + kChunk - 1) / kChunk;
  if (tiles >= (int64_t(1) << 30) || count * chunks >= (int64_t(1) << 30)) return MUON_ERR_SHAPE;
  return MUON_OK;
}

bool finite(float x) { return std::isfinite(x); }

muon_status check_ns(const muon_hparams* hp) {
  if (hp->ns_steps < 1 || hp->ns_steps > MUON_MAX_NS_STEPS) return MUON_ERR_HPARAM;
  for (int i = 0; i < 3 * hp->ns_steps; ++i)
    if (!finite(hp->coeffs[i])) return MUON_ERR_HPARAM;
  if (!finite(hp->eps) || hp->eps < 0.0f) return MUON_ERR_HPARAM;
  return MUON_OK;
}

inline bool beta_ok(float b) { return finite(b) && b >= 0.0f && b < 1.0f; }

bool overlap(const void* a, size_t na, const void* b, size_t nb) {
  if (!a || !b) return false;
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

muon_status check_banks(const muon_bank* banks, int32_t nbanks, bool anvil) {
  if (!banks) return MUON_ERR_NULL;
  if (nbanks < 1 || nbanks > MUON_MAX_BANKS) return MUON_ERR_SHAPE;
  // every buffer the step writes, over all banks: none may overlap another
  const void* bufs[4 * MUON_MAX_BANKS];
  size_t sz[4 * MUON_MAX_BANKS];
  int nb = 0;
  for (int b = 0; b < nbanks; ++b) {
    const muon_bank& k = banks[b];
    muon_status st = check_shape(k.count, k.rows, k.cols);
    if (st != MUON_OK) return st;
    if (!k.param || !k.grad || !k.momentum) return MUON_ERR_NULL;
    if (anvil && !k.momentum_slow) return MUON_ERR_NULL;
    if (!dtype_ok(k.param_dtype) || !dtype_ok(k.grad_dtype)) return MUON_ERR_DTYPE;
    if (!aligned16(k.param) || !aligned16(k.grad) || !aligned16(k.momentum) ||
        !aligned16(k.momentum_slow) || !aligned16(k.ema))
      return MUON_ERR_ALIGN;
    const size_t n = static_cast<size_t>(k.count * k.rows * k.cols);
    const void* w[4] = {k.param, k.momentum, anvil ? k.momentum_slow : nullptr, k.ema};
    const size_t wz[4] = {n * (k.param_dtype == MUON_BF16 ? 2 : 4), n * 4, n * 4, n * 4};
    for (int i = 0; i < 4; ++i) {
      bufs[nb] = w[i];
      sz[nb++] = wz[i];
    }
  }
  for (int i = 0; i < nb; ++i)
    for (int j = i + 1; j < nb; ++j)
      if (overlap(bufs[i], sz[i], bufs[j], sz[j])) return MUON_ERR_ALIAS;
  return MUON_OK;
}

// ------------------------------------------------------------ workspace
struct Shape3 {
  int64_t count, rows, cols;
};

// Returns the workspace bytes needed; fills plans if given (with the buffer
// addresses inside the workspace at base, if base is given).
size_t plan_workspace(const Shape3* shapes, int nbanks, uint8_t* base, BankPlan* plans) {
  size_t off = kHeaderBytes;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 1024);
    return o;
  };
  for (int b = 0; b < nbanks; ++b) {
    const Shape3& s = shapes[b];
    BankPlan p;
    std::memset(&p, 0, sizeof(p));
    p.count = static_cast<int>(s.count);
    p.R = static_cast<int>(s.rows);
    p.C = static_cast<int>(s.cols);
    p.Rp = static_cast<int>(round_up(s.rows, kPad));
    p.Cp = static_cast<int>(round_up(s.cols, kPad));
    p.tall = s.rows > s.cols ? 1 : 0;
    p.rp = p.tall ? p.Cp : p.Rp;
    const size_t padded = static_cast<size_t>(p.Rp) * p.Cp;
    p.chunks = static_cast<int>((padded + kChunk - 1) / kChunk);
    const int nb = p.rp / kTile;
    p.tiles_sym = nb * (nb + 1) / 2;
    p.tiles_apply = (p.Rp / kTile) * (p.Cp / kTile);
    // Split the Gram product along K when the bank has too few Gram tiles to
    // spread and K is much longer than the Gram is wide (e.g. a 768 x 50304
    // readout: 6 tiles of 788 K blocks). Splits keep >= 32 K blocks each.
    const int kg = (p.tall ? p.Rp : p.Cp) / kBK;
    p.ksplit = 1;
    if (p.count * p.tiles_sym < 48 && kg * kBK >= 8 * p.rp) {
      p.ksplit = kg / 32;
      if (p.ksplit > kMaxSplit) p.ksplit = kMaxSplit;
      if (p.ksplit < 1) p.ksplit = 1;
    }
    p.kc = (kg + p.ksplit - 1) / p.ksplit;
    if (p.ksplit > 1) p.ksplit = (kg + p.kc - 1) / p.kc;  // no empty split
    p.tiles_red = p.ksplit > 1 ? p.tiles_sym * kRedSub : 0;
    p.fd_apply = make_fastdiv(p.tiles_apply);
    p.fd_nbn = make_fastdiv(p.Cp / kTile);
    p.fd_gram = make_fastdiv(p.tiles_sym * p.ksplit);
    p.fd_ksplit = make_fastdiv(p.ksplit);
    p.fd_red = make_fastdiv(p.tiles_red);
    p.fd_sym = make_fastdiv(p.tiles_sym);
    const size_t it_bytes = static_cast<size_t>(p.count) * padded * 2;
    const size_t sq_bytes = static_cast<size_t>(p.count) * p.rp * p.rp * 2;
    const size_t o_hi0 = take(it_bytes), o_hi1 = take(it_bytes), o_lo = take(it_bytes);
    const size_t o_A = take(sq_bytes), o_B = take(sq_bytes);
    const size_t o_part = take(static_cast<size_t>(p.count) * p.chunks * 4);
    const size_t o_scale = take(static_cast<size_t>(p.count) * 4);
    const size_t o_cnt = take(static_cast<size_t>(p.count) * 4 * 4);
    const size_t o_gpart = p.ksplit > 1 ? take(static_cast<size_t>(p.count) * p.tiles_sym * p.ksplit *
                                              kTile * kTile * 4)
                                       : 0;
    if (plans) {
      if (!base) {  // geometry only
        plans[b] = p;
        continue;
      }
      p.hi[0] = reinterpret_cast<__nv_bfloat16*>(base + o_hi0);
      p.hi[1] = reinterpret_cast<__nv_bfloat16*>(base + o_hi1);
      p.lo = reinterpret_cast<__nv_bfloat16*>(base + o_lo);
      p.A = reinterpret_cast<__nv_bfloat16*>(base + o_A);
      p.B = reinterpret_cast<__nv_bfloat16*>(base + o_B);
      p.partial = reinterpret_cast<float*>(base + o_part);
      p.scale = reinterpret_cast<float*>(base + o_scale);
      p.counters = reinterpret_cast<int*>(base + o_cnt);
      p.part = p.ksplit > 1 ? reinterpret_cast<float*>(base + o_gpart) : nullptr;
      plans[b] = p;
    }
  }
  return off;
}

muon_status encode_map(CUtensorMap* m, void* ptr, int64_t inner, int64_t outer, int box_inner,
                       int box_outer, CUtensorMapSwizzle swz, bool fp32 = false) {
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(inner) * (fp32 ? 4 : 2)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_outer)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                        2, ptr, dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MUON_OK : MUON_ERR_CUDA;
}

muon_status encode_bank_maps(const BankPlan& p, CUtensorMap* maps) {
  const int64_t rows = static_cast<int64_t>(p.count) * p.Rp;
  const int64_t srows = static_cast<int64_t>(p.count) * p.rp;
  const CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B, sw64 = CU_TENSOR_MAP_SWIZZLE_64B;
  struct Spec {
    int slot;
    void* ptr;
    int64_t inner, outer;
    int bi, bo;
    CUtensorMapSwizzle swz;
  } specs[] = {
      {kHiK0, p.hi[0], p.Cp, rows, 64, 128, sw},    {kHiK1, p.hi[1], p.Cp, rows, 64, 128, sw},
      {kHiMN0, p.hi[0], p.Cp, rows, 64, 64, sw},    {kHiMN1, p.hi[1], p.Cp, rows, 64, 64, sw},
      {kAK, p.A, p.rp, srows, 64, 128, sw},         {kBK_, p.B, p.rp, srows, 64, 128, sw},
      {kHiE0, p.hi[0], p.Cp, rows, kEpiCols, kEpiRows, sw64},
      {kHiE1, p.hi[1], p.Cp, rows, kEpiCols, kEpiRows, sw64},
      {kLoE, p.lo, p.Cp, rows, kEpiCols, kEpiRows, sw64},
      {kAE, p.A, p.rp, srows, kEpiCols, kEpiRows, sw64},
      {kAMN, p.A, p.rp, srows, 64, 64, sw},
      {kBE, p.B, p.rp, srows, kEpiCols, kEpiRows, sw64},
      {kBMN, p.B, p.rp, srows, 64, 64, sw},
  };
  for (const Spec& sp : specs) {
    muon_status st = encode_map(&maps[sp.slot], sp.ptr, sp.inner, sp.outer, sp.bi, sp.bo, sp.swz);
    if (st != MUON_OK) return st;
  }
  if (p.ksplit > 1) {
    const int64_t prow = static_cast<int64_t>(p.count) * p.tiles_sym * p.ksplit * kTile;
    return encode_map(&maps[kPartE], p.part, kTile, prow, kEpiCols, kEpiRows, sw, true);
  }
  return MUON_OK;
}

// ------------------------------------------------------------ the step
enum class Variant { kMuon, kAnvil, kOrtho };

struct OrthoIO {
  const void* in;
  int in_dtype;
  void* out;
  int out_dtype;
};

// The parameter write of a bank: lr times the shape scale max(1, R/C)^(1/2).
UpdBank update_io(const muon_bank& b, const muon_hparams* hp) {
  const double s = std::sqrt(std::fmax(1.0, double(b.rows) / double(b.cols)));
  return UpdBank{b.param, b.param_dtype, b.momentum_slow, b.ema, static_cast<float>(double(hp->lr) * s)};
}

// check_shape bounds each bank on its own; the chain numbers its tiles (over
// every bank, phase and step) and the momentum and update passes their blocks
// (over every bank) with 32-bit ints, so those totals must stay below 2^31.
muon_status check_totals(const Shape3* shapes, int nbanks, int ns_steps) {
  BankPlan plans[MUON_MAX_BANKS];
  plan_workspace(shapes, nbanks, nullptr, plans);
  int64_t tiles = 0, blocks = 0;
  for (int b = 0; b < nbanks; ++b) {
    const BankPlan& p = plans[b];
    tiles += static_cast<int64_t>(p.count) *
             (static_cast<int64_t>(p.tiles_sym) * p.ksplit + p.tiles_red + p.tiles_sym + p.tiles_apply);
    blocks += static_cast<int64_t>(p.count) * p.chunks;
  }
  const int64_t lim = int64_t(1) << 31;
  return (tiles * ns_steps >= lim || blocks >= lim) ? MUON_ERR_SHAPE : MUON_OK;
}

// Tile prefix sums of the chain (list order: step, phase Gram / Reduce / Poly
// / Apply, bank, matrix).
void plan_chain(NsGemmParams& gp, const BankPlan* plans, int nbanks) {
  gp.nbanks = nbanks;
  int gram = 0, red = 0, sym = 0, app = 0;
  for (int b = 0; b < nbanks; ++b) {
    gp.bank[b] = plans[b];
    gp.gram_begin[b] = gram;
    gp.red_begin[b] = red;
    gp.sym_begin[b] = sym;
    gp.apply_begin[b] = app;
    gram += plans[b].count * plans[b].tiles_sym * plans[b].ksplit;
    red += plans[b].count * plans[b].tiles_red;
    sym += plans[b].count * plans[b].tiles_sym;
    app += plans[b].count * plans[b].tiles_apply;
  }
  gp.fd_step = make_fastdiv(static_cast<uint32_t>(gram + red + sym + app));
  gp.gram_begin[nbanks] = gram;
  gp.red_begin[nbanks] = red;
  gp.sym_begin[nbanks] = sym;
  gp.apply_begin[nbanks] = app;
}

muon_status run_step(Variant v, const muon_bank* banks, int nbanks, const muon_hparams* hp,
                     void* ws, size_t ws_bytes, cudaStream_t stream, const OrthoIO* oio) {
  int sms = 0, max_pairs = 0;
  muon_status st = device_state(&sms, &max_pairs);
  if (st != MUON_OK) return st;

  Shape3 shapes[MUON_MAX_BANKS];
  for (int b = 0; b < nbanks; ++b) shapes[b] = {banks[b].count, banks[b].rows, banks[b].cols};
  static thread_local NsGemmParams gp;  // large; kept off the stack
  std::memset(&gp, 0, sizeof(gp));
  BankPlan plans[MUON_MAX_BANKS];
  const size_t need = plan_workspace(shapes, nbanks, static_cast<uint8_t*>(ws), plans);
  if (ws_bytes < need) return MUON_ERR_WORKSPACE;
  int* status = static_cast<int*>(ws);
  // every fallible host-side step comes before the first launch, so an error
  // return means that nothing was enqueued (the momenta are not advanced)
  for (int b = 0; b < nbanks; ++b)
    if ((st = encode_bank_maps(plans[b], gp.maps[b])) != MUON_OK) return st;

  // ---- momentum + norm partials, then 1/(||U||+eps)
  MomParams mp;
  std::memset(&mp, 0, sizeof(mp));
  mp.nbanks = nbanks;
  mp.mode = v == Variant::kMuon ? kMomMuon : (v == Variant::kAnvil ? kMomAnvil : kMomNone);
  mp.mu = v == Variant::kAnvil ? hp->beta_fast : hp->mu;
  mp.mu_slow = hp->beta_slow;
  mp.nesterov = hp->nesterov ? 1 : 0;
  mp.sgd = (v == Variant::kMuon && hp->sgd_momentum) ? 1 : 0;
  mp.eps = hp->eps;
  mp.status = status;
  int blocks = 0, mats = 0;
  for (int b = 0; b < nbanks; ++b) {
    mp.bank[b] = plans[b];
    if (v == Variant::kOrtho) {
      mp.io[b] = {oio->in, nullptr, nullptr, oio->in_dtype};
    } else {
      mp.io[b] = {banks[b].grad, banks[b].momentum, banks[b].momentum_slow, banks[b].grad_dtype};
    }
    mp.block_begin[b] = blocks;
    mp.mat_begin[b] = mats;
    blocks += plans[b].count * plans[b].chunks;
    mats += plans[b].count;
  }
  mp.block_begin[nbanks] = blocks;
  mp.mat_begin[nbanks] = mats;
  if (launch_momentum_norm(mp, blocks, mats, stream) != cudaSuccess) return MUON_ERR_CUDA;

  // ---- Newton-Schulz chain
  gp.status = status;
  const double lim = g_debug.wait_limit_s > 0 ? g_debug.wait_limit_s : 2.0;
  gp.wait_limit_ns = static_cast<unsigned long long>(lim * 1e9);
  gp.fault = g_debug.fault;
  cudaEvent_t ev_before = nullptr, ev_after = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    std::swap(ev_before, g_ev_before);
    std::swap(ev_after, g_ev_after);
  }
  if (ev_before && cudaEventRecord(ev_before, stream) != cudaSuccess) return MUON_ERR_CUDA;
  gp.ns_steps = hp->ns_steps;
  gp.keep_lo = v == Variant::kOrtho ? 1 : 0;
  for (int i = 0; i < 3 * hp->ns_steps; ++i) gp.coef[i] = hp->coeffs[i];
  plan_chain(gp, plans, nbanks);
  if (launch_ns_gemm(gp, max_pairs, stream) != cudaSuccess) return MUON_ERR_CUDA;
  if (ev_after && cudaEventRecord(ev_after, stream) != cudaSuccess) return MUON_ERR_CUDA;

  // ---- scale, decay, parameter write (+ EMA), or O out
  UpdParams up;
  std::memset(&up, 0, sizeof(up));
  up.nbanks = nbanks;
  up.mode = v == Variant::kMuon ? kUpdDecoupled : (v == Variant::kAnvil ? kUpdCautious : kUpdWriteO);
  up.final_buf = hp->ns_steps & 1;
  up.use_lo = v == Variant::kOrtho ? 1 : 0;
  up.lr_wd = hp->lr * hp->weight_decay;
  up.ema_beta = hp->ema_beta;
  up.status = status;
  for (int b = 0; b < nbanks; ++b) {
    up.bank[b] = plans[b];
    if (v == Variant::kOrtho) {
      up.io[b] = {oio->out, oio->out_dtype, nullptr, nullptr, 0.0f};
    } else {
      up.io[b] = update_io(banks[b], hp);
    }
    up.block_begin[b] = mp.block_begin[b];
  }
  up.block_begin[nbanks] = mp.block_begin[nbanks];
  if (launch_update(up, mp.block_begin[nbanks], stream) != cudaSuccess) return MUON_ERR_CUDA;
  return MUON_OK;
}

muon_status check_common(const muon_bank* banks, int32_t nbanks, const muon_hparams* hp, void* ws,
                         bool anvil) {
  if (!hp) return MUON_ERR_NULL;
  muon_status st = check_banks(banks, nbanks, anvil);
  if (st != MUON_OK) return st;
  if ((st = check_ns(hp)) != MUON_OK) return st;
  Shape3 shapes[MUON_MAX_BANKS];
  for (int b = 0; b < nbanks; ++b) shapes[b] = {banks[b].count, banks[b].rows, banks[b].cols};
  if ((st = check_totals(shapes, nbanks, hp->ns_steps)) != MUON_OK) return st;
  if (!finite(hp->lr) || !finite(hp->weight_decay) || hp->weight_decay < 0.0f) return MUON_ERR_HPARAM;
  if (anvil) {
    if (!beta_ok(hp->beta_fast) || !beta_ok(hp->beta_slow)) return MUON_ERR_HPARAM;
  } else if (!beta_ok(hp->mu)) {
    return MUON_ERR_HPARAM;
  }
  for (int b = 0; b < nbanks; ++b)
    if (banks[b].ema && !beta_ok(hp->ema_beta)) return MUON_ERR_HPARAM;
  if (!ws) return MUON_ERR_WORKSPACE;
  if (!aligned16(ws)) return MUON_ERR_ALIGN;
  return MUON_OK;
}

}  // namespace

extern "C" {

int32_t muon_abi_version(void) { return MUON_ABI_VERSION; }

const char* muon_status_string(muon_status s) {
  switch (s) {
    case MUON_OK: return "MUON_OK";
    case MUON_ERR_NULL: return "MUON_ERR_NULL: a required pointer is NULL";
    case MUON_ERR_SHAPE: return "MUON_ERR_SHAPE: bad count/rows/cols or number of banks";
    case MUON_ERR_DTYPE: return "MUON_ERR_DTYPE: unsupported dtype";
    case MUON_ERR_ALIGN: return "MUON_ERR_ALIGN: pointer not 16-byte aligned";
    case MUON_ERR_HPARAM: return "MUON_ERR_HPARAM: hyper-parameter out of range";
    case MUON_ERR_WORKSPACE: return "MUON_ERR_WORKSPACE: workspace missing or too small";
    case MUON_ERR_CUDA: return "MUON_ERR_CUDA: CUDA runtime error";
    case MUON_ERR_TIMEOUT: return "MUON_ERR_TIMEOUT: a bounded device wait ran out";
    case MUON_ERR_ALIAS: return "MUON_ERR_ALIAS: in-place buffers overlap";
    case MUON_ERR_BOUNDS: return "MUON_ERR_BOUNDS: an index outside its buffer (debug build)";
  }
  return "unknown muon_status";
}

size_t muon_workspace_size(const muon_bank* banks, int32_t nbanks) {
  if (!banks || nbanks < 1 || nbanks > MUON_MAX_BANKS) return 0;
  Shape3 shapes[MUON_MAX_BANKS];
  for (int b = 0; b < nbanks; ++b) {
    if (check_shape(banks[b].count, banks[b].rows, banks[b].cols) != MUON_OK) return 0;
    shapes[b] = {banks[b].count, banks[b].rows, banks[b].cols};
  }
  return plan_workspace(shapes, nbanks, nullptr, nullptr);
}

muon_status muon_step(const muon_bank* banks, int32_t nbanks, const muon_hparams* hp, void* ws,
                      size_t ws_bytes, void* stream) {
  muon_status st = check_common(banks, nbanks, hp, ws, false);
  if (st != MUON_OK) return st;
  if (ws_bytes < muon_workspace_size(banks, nbanks)) return MUON_ERR_WORKSPACE;
  return run_step(Variant::kMuon, banks, nbanks, hp, ws, ws_bytes,
                  static_cast<cudaStream_t>(stream), nullptr);
}

muon_status anvil_step(const muon_bank* banks, int32_t nbanks, const muon_hparams* hp, void* ws,
                       size_t ws_bytes, void* stream) {
  muon_status st = check_common(banks, nbanks, hp, ws, true);
  if (st != MUON_OK) return st;
  if (ws_bytes < muon_workspace_size(banks, nbanks)) return MUON_ERR_WORKSPACE;
  return run_step(Variant::kAnvil, banks, nbanks, hp, ws, ws_bytes,
                  static_cast<cudaStream_t>(stream), nullptr);
}

muon_status muon_orthogonalize(const void* in, int32_t in_dtype, void* out, int32_t out_dtype,
                               int64_t count, int64_t rows, int64_t cols, const muon_hparams* hp,
                               void* ws, size_t ws_bytes, void* stream) {
  if (!in || !out || !hp) return MUON_ERR_NULL;
  muon_status st = check_shape(count, rows, cols);
  if (st != MUON_OK) return st;
  if (!dtype_ok(in_dtype) || !dtype_ok(out_dtype)) return MUON_ERR_DTYPE;
  if (!aligned16(in) || !aligned16(out)) return MUON_ERR_ALIGN;
  if ((st = check_ns(hp)) != MUON_OK) return st;
  const Shape3 one = {count, rows, cols};
  if ((st = check_totals(&one, 1, hp->ns_steps)) != MUON_OK) return st;
  if (!ws) return MUON_ERR_WORKSPACE;
  if (!aligned16(ws)) return MUON_ERR_ALIGN;
  muon_bank bank;
  std::memset(&bank, 0, sizeof(bank));
  bank.count = count;
  bank.rows = rows;
  bank.cols = cols;
  if (ws_bytes < muon_workspace_size(&bank, 1)) return MUON_ERR_WORKSPACE;
  const size_t n = static_cast<size_t>(count * rows * cols);
  if (overlap(in, n * (in_dtype == MUON_BF16 ? 2 : 4), out, n * (out_dtype == MUON_BF16 ? 2 : 4)))
    return MUON_ERR_ALIAS;
  OrthoIO io{in, in_dtype, out, out_dtype};
  return run_step(Variant::kOrtho, &bank, 1, hp, ws, ws_bytes, static_cast<cudaStream_t>(stream),
                  &io);
}

muon_status ema_update(const muon_bank* banks, int32_t nbanks, float beta, void* stream) {
  if (!banks) return MUON_ERR_NULL;
  if (nbanks < 1 || nbanks > MUON_MAX_BANKS) return MUON_ERR_SHAPE;
  if (!beta_ok(beta)) return MUON_ERR_HPARAM;
  for (int b = 0; b < nbanks; ++b) {
    const muon_bank& k = banks[b];
    if (!k.ema) continue;
    if (check_shape(k.count, k.rows, k.cols) != MUON_OK) return MUON_ERR_SHAPE;
    if (!k.param) return MUON_ERR_NULL;
    if (!dtype_ok(k.param_dtype)) return MUON_ERR_DTYPE;
    if (!aligned16(k.param) || !aligned16(k.ema)) return MUON_ERR_ALIGN;
  }
  int sms = 0;
  muon_status st = device_state(&sms);
  if (st != MUON_OK) return st;
  for (int b = 0; b < nbanks; ++b) {
    const muon_bank& k = banks[b];
    if (!k.ema) continue;
    if (launch_ema(k.ema, k.param, k.param_dtype, k.count * k.rows * k.cols, beta, sms,
                   static_cast<cudaStream_t>(stream)) != cudaSuccess)
      return MUON_ERR_CUDA;
  }
  return MUON_OK;
}

muon_status readout_blend(const void* theta, int32_t theta_dtype, const float* ema, void* out,
                          int32_t out_dtype, int64_t n, float w_final, void* stream) {
  if (!theta || !ema || !out) return MUON_ERR_NULL;
  if (n < 1) return MUON_ERR_SHAPE;
  if (!dtype_ok(theta_dtype) || !dtype_ok(out_dtype)) return MUON_ERR_DTYPE;
  if (!aligned16(theta) || !aligned16(ema) || !aligned16(out)) return MUON_ERR_ALIGN;
  if (!finite(w_final)) return MUON_ERR_HPARAM;
  int sms = 0;
  muon_status st = device_state(&sms);
  if (st != MUON_OK) return st;
  if (launch_blend(theta, theta_dtype, ema, out, out_dtype, n, w_final, sms,
                   static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MUON_ERR_CUDA;
  return MUON_OK;
}

muon_status muon_device_status(void* ws, size_t ws_bytes, void* stream, int32_t clear) {
  if (!ws) return MUON_ERR_NULL;
  if (ws_bytes < kHeaderBytes) return MUON_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int v = 0;
  if (cudaMemcpyAsync(&v, ws, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return MUON_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MUON_ERR_CUDA;
  if (clear) {
    if (cudaMemsetAsync(ws, 0, sizeof(int), s) != cudaSuccess) return MUON_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return MUON_ERR_CUDA;
  }
  return v == 0 ? MUON_OK : static_cast<muon_status>(v);
}

}  // extern "C"

// ------------------------------------------------- fixed scratch, no allocation
// Scratch for muon_orthogonalize_static: one file-scope device array. Host code
// must not use its name as a device address; the address is looked up once per
// device with cudaGetSymbolAddress, with that device current.
static __device__ __align__(256) unsigned char g_static_scratch[MUON_STATIC_SCRATCH_BYTES];

namespace {
void* g_static_ptr[64] = {};

muon_status static_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MUON_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_static_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr)
      return MUON_ERR_CUDA;
    g_static_ptr[dev] = p;
  }
  *out = g_static_ptr[dev];
  return MUON_OK;
}
}  // namespace

extern "C" {

muon_status muon_orthogonalize_static(const void* in, int32_t in_dtype, void* out,
                                      int32_t out_dtype, int64_t count, int64_t rows,
                                      int64_t cols, const muon_hparams* hp, void* stream) {
  if (!in || !out || !hp) return MUON_ERR_NULL;
  muon_status st = check_shape(count, rows, cols);
  if (st != MUON_OK) return st;
  if (!dtype_ok(in_dtype) || !dtype_ok(out_dtype)) return MUON_ERR_DTYPE;
  if (!aligned16(in) || !aligned16(out)) return MUON_ERR_ALIGN;
  if ((st = check_ns(hp)) != MUON_OK) return st;
  const Shape3 one = {count, rows, cols};
  if ((st = check_totals(&one, 1, hp->ns_steps)) != MUON_OK) return st;
  muon_bank bank;
  std::memset(&bank, 0, sizeof(bank));
  bank.count = count;
  bank.rows = rows;
  bank.cols = cols;
  const size_t need = muon_workspace_size(&bank, 1);
  if (need == 0 || need > MUON_STATIC_SCRATCH_BYTES) return MUON_ERR_WORKSPACE;
  const size_t n = static_cast<size_t>(count * rows * cols);
  if (overlap(in, n * (in_dtype == MUON_BF16 ? 2 : 4), out, n * (out_dtype == MUON_BF16 ? 2 : 4)))
    return MUON_ERR_ALIAS;
  void* ws = nullptr;
  if ((st = static_scratch(&ws)) != MUON_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the status word is the only part of the scratch that must start at zero
  if (cudaMemsetAsync(ws, 0, sizeof(int), s) != cudaSuccess) return MUON_ERR_CUDA;
  OrthoIO io{in, in_dtype, out, out_dtype};
  return run_step(Variant::kOrtho, &bank, 1, hp, ws, MUON_STATIC_SCRATCH_BYTES, s, &io);
}

muon_status muon_set_ns_events(void* before_ns, void* after_ns) {
  if ((before_ns == nullptr) != (after_ns == nullptr)) return MUON_ERR_NULL;
  std::lock_guard<std::mutex> lk(g_mu);
  g_ev_before = static_cast<cudaEvent_t>(before_ns);
  g_ev_after = static_cast<cudaEvent_t>(after_ns);
  return MUON_OK;
}

int64_t muon_chain_plan(const int64_t* shapes, int32_t nbanks, int32_t ns_steps, int32_t* tiles,
                        int64_t tiles_cap) {
  if (!shapes) return -static_cast<int64_t>(MUON_ERR_NULL);
  if (nbanks < 1 || nbanks > MUON_MAX_BANKS) return -static_cast<int64_t>(MUON_ERR_SHAPE);
  if (ns_steps < 1 || ns_steps > MUON_MAX_NS_STEPS) return -static_cast<int64_t>(MUON_ERR_HPARAM);
  Shape3 sh[MUON_MAX_BANKS];
  for (int b = 0; b < nbanks; ++b) {
    sh[b] = {shapes[3 * b], shapes[3 * b + 1], shapes[3 * b + 2]};
    const muon_status st = check_shape(sh[b].count, sh[b].rows, sh[b].cols);
    if (st != MUON_OK) return -static_cast<int64_t>(st);
  }
  const muon_status tot = check_totals(sh, nbanks, ns_steps);
  if (tot != MUON_OK) return -static_cast<int64_t>(tot);
  static thread_local NsGemmParams gp;  // large; kept off the stack
  std::memset(&gp, 0, sizeof(gp));
  BankPlan plans[MUON_MAX_BANKS];
  plan_workspace(sh, nbanks, nullptr, plans);
  plan_chain(gp, plans, nbanks);
  gp.ns_steps = ns_steps;
  const int64_t nt = static_cast<int64_t>(ns_steps) * tiles_per_step(gp);
  if (tiles && tiles_cap >= 13 * nt)
    for (int64_t t = 0; t < nt; ++t) {
      const Tile T = decode_tile(gp, static_cast<int>(t));
      int32_t* o = tiles + 13 * t;
      o[0] = T.iter; o[1] = T.phase; o[2] = T.bank; o[3] = T.mat; o[4] = T.m0; o[5] = T.n0;
      o[6] = T.kb0; o[7] = T.nkb; o[8] = T.a_map; o[9] = T.a_base; o[10] = T.b_map; o[11] = T.b_base;
      o[12] = T.same_ab;
    }
  return nt;
}

muon_status muon_set_debug(int32_t fault_mode, double wait_limit_seconds) {
  if (fault_mode < 0 || fault_mode > 1) return MUON_ERR_HPARAM;
  std::lock_guard<std::mutex> lk(g_mu);
  g_debug.fault = fault_mode;
  g_debug.wait_limit_s = wait_limit_seconds > 0 ? wait_limit_seconds : 2.0;
  return MUON_OK;
}

}  // extern "C"
