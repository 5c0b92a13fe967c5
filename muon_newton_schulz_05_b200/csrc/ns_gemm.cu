// Newton-Schulz GEMM chain on sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// One persistent launch runs the whole chain: every step and phase of every
// matrix of every bank (see NsGemmParams). The three phases of a step are
//   Gram : A = X X^T            (tall: A = Y^T Y)      upper 256-blocks only
//   Poly : B = b A + c A A      (A symmetric)          upper 256-blocks only
//   Apply: X <- a X + B X       (tall: Y <- a Y + Y B) full tiles
// A and B keep only their upper 256 x 256 blocks (diagonal blocks whole); an
// operand block below the diagonal is read from the stored block across it,
// as an MN-major (transposed) operand.
// ("Muonとは" / "Muonが登場": approximate orthogonalisation by Newton-Schulz
// iteration, bf16 operands; the polynomial step is the method statement's.)
//
// CTA pairs (clusters of 2 on one TPC) compute 256 x 256 output tiles with the
// 2-SM MMA (tcgen05.mma.cta_group::2, M = 256, N = 256, K = 16): each CTA
// stages its own 128 rows of the A operand and its half (128 rows) of the B
// operand, so every SM reads 32 KB per 64-deep K step instead of 48 KB (16 KB
// on the diagonal blocks of Gram and Poly, where the two operands coincide).
// No TMA multicast is used; only the MMA commits arrive on both CTAs.
//
// Block layout (320 threads, one block per SM), in both CTAs of a pair:
//   warp 0     one thread issues this CTA's TMA loads into a kStages-deep
//              ring; completion is counted on the even (leader) CTA's barrier
//   warp 1     allocates 512 TMEM columns (pair allocation); in the leader one
//              thread issues the MMAs into one of two 256-column accumulators
//   warps 2..9 epilogue: tcgen05.ld this CTA's 128 accumulator rows (warp w
//              reads TMEM lanes 32*(w%4)..+31; two warps per lane quadrant
//              split the 256 columns), apply the phase's axpy and store;
//              the accumulator goes back to the MMA as soon as its last
//              columns are in registers, and the CTA's part of a tile is
//              published one tile later by the last warp to confirm it
// The epilogue of tile t overlaps the MMAs of tile t+1 through the two
// accumulators. Every wait is bounded (muon::mbar_wait*).
#include <cuda_runtime.h>

#include "plan.cuh"
#include "ptx.cuh"
#include "tiles.cuh"


namespace muon {


// Bounded wait until *cnt >= target (acquire, GPU scope), then order the
// async-proxy (TMA) reads that follow after it. False if it gave up.
__device__ __forceinline__ bool wait_dependency(const int* cnt, int target, volatile int* abort,
                                                int* status, uint64_t limit_ns) {
  if (target > 0 && ld_acquire_gpu(cnt) < target) {
    const uint64_t t0 = global_timer_ns();
    for (uint32_t i = 1;; ++i) {
      __nanosleep(64);
      if (ld_acquire_gpu(cnt) >= target) break;
      if ((i & 15u) == 0) {
        // another CTA's wait ran out (or an earlier launch's): the counter may
        // never reach the target, so give up at once
        if (*abort || *reinterpret_cast<volatile int*>(status)) {
          *abort = 1;
          return false;
        }
        if (global_timer_ns() - t0 > limit_ns) {
          *abort = 1;
          atomicExch(status, 8 /* MUON_ERR_TIMEOUT */);
          return false;
        }
      }
    }
  }
  fence_proxy_async_global();
  return true;
}

// This CTA's 128 (MN) x 64 (K) slice of an operand tile into dst; completion
// is counted on the pair leader's barrier bar (shared::cluster address).
//  K-major : one box of 128 rows x 64 K (16 KB).
//  MN-major: two boxes of 64 K rows x 64 MN (8 KB each), stacked along MN.
__device__ __forceinline__ void load_operand(uint8_t* dst, const CUtensorMap* map, uint32_t bar,
                                             int mn_major, int base, int mn0, int k0) {
  if (!mn_major) {
    tma_load_2d_pair(dst, map, bar, k0, base + mn0);
  } else {
    tma_load_2d_pair(dst, map, bar, mn0, base + k0);
    tma_load_2d_pair(dst + 8192, map, bar, mn0 + 64, base + k0);
  }
}

// Debug build: the boxes load_operand would copy lie inside their tensor map
// (X maps: Cp columns x count*Rp rows; A and B maps: rp x count*rp). On a
// violation the status word gets MUON_ERR_BOUNDS and the caller loads from
// (0, 0) instead, so that the stage's bytes still arrive. Release build: true.
__device__ __forceinline__ bool operand_in_bounds(const NsGemmParams& p, const BankPlan& bp, int slot,
                                                  int mn_major, int base, int mn0, int k0) {
  const bool x_map = slot == kHiK0 || slot == kHiK1 || slot == kHiMN0 || slot == kHiMN1;
  const int64_t inner = x_map ? bp.Cp : bp.rp;
  const int64_t outer = static_cast<int64_t>(bp.count) * (x_map ? bp.Rp : bp.rp);
  const bool ok = mn_major ? (mn0 >= 0 && mn0 + 128 <= inner && base + k0 >= 0 && base + k0 + kBK <= outer)
                           : (k0 >= 0 && k0 + kBK <= inner && base + mn0 >= 0 && base + mn0 + kBM <= outer);
  return in_bounds(ok, p.status);
}

// Whether K block k0 of an operand whose rows start at mn0 is read
// transposed: the operand is A or B and the 256-block (mn0, k0) lies below
// the diagonal, so its values are those of the stored block (k0, mn0).
__device__ __forceinline__ bool below_diagonal(int sym, int mn0, int k0) {
  return sym && k0 / kTile < mn0 / kTile;
}

__device__ __forceinline__ uint64_t operand_desc(uint32_t tile_addr, int mn_major, int ks) {
  return mn_major ? smem_desc_sw128(tile_addr + ks * 2048, 8192, 1024)
                  : smem_desc_sw128(tile_addr + ks * 32, 16, 1024);
}

// ---------------------------------------------------------------- epilogues
// Each epilogue warp owns 32 accumulator rows and 128 of the 256 columns and
// works through them in 32 x 32 chunks. Global traffic goes through TMA only,
// through kEpiBufs chunk buffers per warp: the bulk loads of a tile's first
// chunks (Apply: hi and lo of the iterate; Poly: A) are issued when the tile
// starts, while its MMAs run, and the stores of earlier chunks drain while
// later ones are computed. (Loading the next tile's first chunks while the
// current one is still being worked on measured slower: those loads compete
// with the operand loads the tensor cores are waiting for.) Halves use the
// 64-byte swizzle of the TMA box (16-byte group g of
// row r at r*64 + ((g ^ ((r >> 1) & 3)) * 16)), so a lane reading or writing
// its own row touches 8 distinct bank groups per quarter warp.
__device__ __forceinline__ uint32_t swz64_off(int r, int g) {
  return static_cast<uint32_t>(r * 64 + ((g ^ ((r >> 1) & 3)) << 4));
}

// Ring positions: every chunk this warp handles takes the next position k;
// position k uses buffer k % kEpiBufs and load barrier k % kEpiBufs. A load
// for position k is issued once position k - kEpiBufs has had its store read
// out of the buffer.
struct EpiRing {
  uint8_t* base;     // kEpiBufs buffers of kEpiChunkBytes (two halves each)
  uint64_t* bar;     // kEpiBufs load barriers
  uint32_t parity;   // bit i: parity of the next completion of bar[i]
  uint32_t chunk;    // chunks handled so far by this warp (ring position)
  uint32_t inflight; // lane 0: bit i set while a load into buffer i is outstanding
};

__device__ __forceinline__ uint8_t* ring_buf(const EpiRing& e, uint32_t k) {
  return e.base + (k % kEpiBufs) * kEpiChunkBytes;
}

// The epilogue of Apply (hi and lo of the iterate) and Poly (A) tiles reads
// inputs; Gram tiles only store.
__device__ __forceinline__ bool epi_has_loads(const Tile& T) {
  return T.phase == kApply || T.phase == kPoly;
}

// Non-blocking: has the phase this tile reads finished (acquire, GPU scope)?
__device__ __forceinline__ bool dependency_met(const Tile& T) {
  return T.dep_target <= 0 || ld_acquire_gpu(T.dep_cnt) >= T.dep_target;
}

// Lane 0 issues the bulk loads of ring chunk k (column c0 of this warp's rows).
__device__ __forceinline__ void epi_issue_load(const NsGemmParams& p, EpiRing& e,
                                               const Tile& T, const BankPlan& bp, int r0, int c0,
                                               uint32_t k) {
  uint8_t* b = ring_buf(e, k);
  uint64_t* bar = &e.bar[k % kEpiBufs];
  e.inflight |= 1u << (k % kEpiBufs);
  if (T.phase == kApply) {
    const int y = T.mat * bp.Rp + r0;
    if (!in_bounds(T.mat < bp.count && r0 + kEpiRows <= bp.Rp && c0 + kEpiCols <= bp.Cp, p.status)) {
      mbar_arrive_expect_tx(bar, 0);  // debug build: no copy, the wait still completes
      return;
    }
    mbar_arrive_expect_tx(bar, kEpiChunkBytes);
    tma_load_2d(b, &p.maps[T.bank][kHiE0 + T.cur], bar, c0, y);
    tma_load_2d(b + kEpiHalfBytes, &p.maps[T.bank][kLoE], bar, c0, y);
  } else if (T.phase == kPoly) {
    if (!in_bounds(T.mat < bp.count && r0 + kEpiRows <= bp.rp && c0 + kEpiCols <= bp.rp, p.status)) {
      mbar_arrive_expect_tx(bar, 0);
      return;
    }
    mbar_arrive_expect_tx(bar, kEpiHalfBytes);
    tma_load_2d(b, &p.maps[T.bank][kAE], bar, c0, T.mat * bp.rp + r0);
  }
}

// Chunk j (of kChunks) of tile X for this warp: lane 0 issues its loads into
// ring position k.
__device__ __forceinline__ void epi_issue_chunk(const NsGemmParams& p, EpiRing& e, const Tile& X,
                                                int rank, int q, int half, int j, uint32_t k) {
  const BankPlan& bp = p.bank[X.bank];
  epi_issue_load(p, e, X, bp, X.m0 + kBM * rank + 32 * q, X.n0 + half * 128 + j * kEpiCols, k);
}

// Every lane waits for ring chunk k's loads. False if the wait gave up (the
// load then still counts as outstanding, so that it can be drained).
__device__ __forceinline__ bool epi_wait_load(const NsGemmParams& p, EpiRing& e, uint32_t k,
                                              volatile int* abort_flag) {
  const uint32_t i = k % kEpiBufs;
  const bool ok = __all_sync(0xffffffffu, mbar_wait(&e.bar[i], (e.parity >> i) & 1u, abort_flag,
                                                    p.status, p.wait_limit_ns));
  if (ok) {
    e.parity ^= 1u << i;
    e.inflight &= ~(1u << i);
  }
  return ok;
}

// This warp's stores of a tile are complete (the caller waited for its bulk
// groups): count it in the CTA's slot for that tile. The warp that completes
// the count publishes the CTA's part of the tile with one release, so no
// warp waits for another. Slot counters only grow; the tile's last arrival
// is the one that makes the count a multiple of kEpiWarps. A slot is reused
// four tiles later, after every warp has confirmed the tile that used it.
__device__ __forceinline__ void confirm_tile(uint32_t* slot_count, int* done_cnt) {
  static_assert((kEpiWarps & (kEpiWarps - 1)) == 0, "kEpiWarps must be a power of two");
  fence_proxy_async_global();
  if ((atom_add_acq_rel_cta(slot_count, 1u) & (kEpiWarps - 1)) == kEpiWarps - 1)
    red_release_gpu_add(done_cnt, 1);
}

// Apply: x' = alpha x + beta D with x = hi + lo, for this lane's row.
__device__ __forceinline__ void epi_apply(const Tile& T, const BankPlan& bp, uint8_t* buf, int lane,
                                          const uint32_t (&r)[32]) {
  float alpha = T.a, beta = 1.0f;
  if (T.iter == 0) {  // the iterate holds U; X0 = s U
    const float s = bp.scale[T.mat];
    alpha *= s;
    beta = s;
  }
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    const uint32_t off = swz64_off(lane, g);
    const uint4 h4 = *reinterpret_cast<const uint4*>(buf + off);
    const uint4 l4 = *reinterpret_cast<const uint4*>(buf + kEpiHalfBytes + off);
    const uint32_t hw[4] = {h4.x, h4.y, h4.z, h4.w};
    const uint32_t lw[4] = {l4.x, l4.y, l4.z, l4.w};
    uint32_t ho[4], lo[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const float y0 = fmaf(alpha, bf16_lo_f(hw[h]) + bf16_lo_f(lw[h]), beta * __uint_as_float(r[8 * g + 2 * h]));
      const float y1 = fmaf(alpha, bf16_hi_f(hw[h]) + bf16_hi_f(lw[h]), beta * __uint_as_float(r[8 * g + 2 * h + 1]));
      ho[h] = pack_bf16x2(y0, y1);
      lo[h] = pack_bf16x2(y0 - bf16_lo_f(ho[h]), y1 - bf16_hi_f(ho[h]));
    }
    *reinterpret_cast<uint4*>(buf + off) = make_uint4(ho[0], ho[1], ho[2], ho[3]);
    *reinterpret_cast<uint4*>(buf + kEpiHalfBytes + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
  }
}

// Gram (A = D, times s^2 at step 0) or Poly (B = b A + c D) for this lane's row.
__device__ __forceinline__ void epi_sym(const Tile& T, const BankPlan& bp, uint8_t* buf, int lane,
                                        const uint32_t (&r)[32]) {
  float scl = 1.0f;
  if (T.phase != kPoly && T.iter == 0) {  // Gram / Reduce of U: fold 1 / ||U||^2 in here
    const float s = bp.scale[T.mat];
    scl = s * s;
  }
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    const uint32_t off = swz64_off(lane, g);
    float v[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) v[t] = __uint_as_float(r[8 * g + t]);
    if (T.phase == kPoly) {
      const uint4 a4 = *reinterpret_cast<const uint4*>(buf + off);
      const uint32_t aw[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        v[2 * h] = fmaf(T.c, v[2 * h], T.b * bf16_lo_f(aw[h]));
        v[2 * h + 1] = fmaf(T.c, v[2 * h + 1], T.b * bf16_hi_f(aw[h]));
      }
    } else {
#pragma unroll
      for (int t = 0; t < 8; ++t) v[t] *= scl;
    }
    uint32_t pk[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) pk[h] = pack_bf16x2(v[2 * h], v[2 * h + 1]);
    *reinterpret_cast<uint4*>(buf + off) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  }
}

// Bulk-store ring chunk k (lane 0, after every lane's writes are visible to
// the async proxy) as one bulk group.
__device__ __forceinline__ void epi_store(const NsGemmParams& p, const Tile& T, const BankPlan& bp,
                                          uint8_t* buf, int r0, int c0, int lane) {
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    const int rows = T.phase == kApply ? bp.Rp : bp.rp, cols = T.phase == kApply ? bp.Cp : bp.rp;
    if (!in_bounds(T.mat < bp.count && r0 + kEpiRows <= rows && c0 + kEpiCols <= cols, p.status)) {
      bulk_commit();  // debug build: the chunk is not stored (an empty bulk group)
      return;
    }
    if (T.phase == kApply) {
      const int y = T.mat * bp.Rp + r0;
      tma_store_2d(&p.maps[T.bank][kHiE0 + (T.cur ^ 1)], buf, c0, y);
      // the parameter update takes O in bf16; the low part of the last
      // iterate is stored only when O itself is the requested output
      if (T.iter + 1 < p.ns_steps || p.keep_lo)
        tma_store_2d(&p.maps[T.bank][kLoE], buf + kEpiHalfBytes, c0, y);
    } else {
      const int base = T.mat * bp.rp;
      tma_store_2d(&p.maps[T.bank][T.phase == kPoly ? kBE : kAE], buf, c0, base + r0);
    }
    bulk_commit();
  }
}

// ------------------------------------------------- split Gram: partials, Reduce
// fp32 chunk buffers use the 128-byte swizzle of a 32 x 32 fp32 box: 16-byte
// group g of row r at r*128 + ((g ^ (r & 7)) * 16).
__device__ __forceinline__ uint32_t swz128_off(int r, int g) {
  return static_cast<uint32_t>(r * 128 + ((g ^ (r & 7)) << 4));
}

// Split Gram tile: this lane's row of the fp32 partial chunk goes to the
// buffer, then the chunk is bulk-stored at (pcol, prow) of the partial map.
__device__ __forceinline__ void epi_partial(const NsGemmParams& p, const Tile& T, uint8_t* buf,
                                            int lane, int prow, int pcol, const uint32_t (&r)[32]) {
#pragma unroll
  for (int g = 0; g < 8; ++g)
    *reinterpret_cast<uint4*>(buf + swz128_off(lane, g)) =
        make_uint4(r[4 * g], r[4 * g + 1], r[4 * g + 2], r[4 * g + 3]);
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(&p.maps[T.bank][kPartE], buf, pcol, prow);
    bulk_commit();
  }
}

// Reduce sub-tile: this warp sums the ksplit partials of its 32 x 32 chunk in
// split order (deterministic), folds in 1/||U||^2 at step 0, and stores the
// bf16 chunk of A. Requires every earlier
// bulk store of the warp to be complete (all ring buffers free). False if a
// wait gave up.
__device__ __forceinline__ bool epi_reduce(const NsGemmParams& p, EpiRing& e, const Tile& T,
                                           const BankPlan& bp, int lane, int rank, int q, int half,
                                           volatile int* abort_flag) {
  const int ks = bp.ksplit;
  const int prow0 = (T.mat * bp.tiles_sym + T.sym_t) * ks * kTile + kBM * rank + 32 * q;
  const int pcol = half * 128 + kEpiCols * T.sub;
  const CUtensorMap* pmap = &p.maps[T.bank][kPartE];
  constexpr int kAhead = kEpiBufs - 1;  // partials in flight beyond the one being summed
  if (lane == 0) {
    for (int s = 0; s < kAhead && s < ks; ++s) {
      e.inflight |= 1u << s;
      mbar_arrive_expect_tx(&e.bar[s], kEpiChunkBytes);
      tma_load_2d(e.base + s * kEpiChunkBytes, pmap, &e.bar[s], pcol, prow0 + s * kTile);
    }
  }
  float acc[32];
#pragma unroll
  for (int t = 0; t < 32; ++t) acc[t] = 0.0f;
  for (int s = 0; s < ks; ++s) {
    // partial s+kAhead goes to the buffer of partial s-1, which every lane has summed
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0 && s + kAhead < ks) {
      const int slot = (s + kAhead) % kEpiBufs;
      e.inflight |= 1u << slot;
      mbar_arrive_expect_tx(&e.bar[slot], kEpiChunkBytes);
      tma_load_2d(e.base + slot * kEpiChunkBytes, pmap, &e.bar[slot], pcol, prow0 + (s + kAhead) * kTile);
    }
    const int slot = s % kEpiBufs;
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&e.bar[slot], (e.parity >> slot) & 1u,
                                                      abort_flag, p.status, p.wait_limit_ns));
    if (!ok) return false;  // the load stays outstanding, to be drained
    e.parity ^= 1u << slot;
    e.inflight &= ~(1u << slot);
    const uint8_t* b = e.base + slot * kEpiChunkBytes;
#pragma unroll
    for (int g = 0; g < 8; ++g) {
      const float4 v = *reinterpret_cast<const float4*>(b + swz128_off(lane, g));
      acc[4 * g] += v.x;
      acc[4 * g + 1] += v.y;
      acc[4 * g + 2] += v.z;
      acc[4 * g + 3] += v.w;
    }
  }
  static_assert(kEpiBufs >= 2, "the Reduce loop keeps one partial in flight");
  __syncwarp();
  uint32_t bits[32];
#pragma unroll
  for (int t = 0; t < 32; ++t) bits[t] = __float_as_uint(acc[t]);
  uint8_t* buf = e.base;  // every load has been consumed
  const int r0 = T.m0 + kBM * rank + 32 * q;
  const int c0 = T.n0 + half * 128 + kEpiCols * T.sub;
  epi_sym(T, bp, buf, lane, bits);
  epi_store(p, T, bp, buf, r0, c0, lane);
  return true;
}

// Waits that ignore the abort flag, used only to drain in-flight work.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  const uint32_t addr = smem_u32(bar);
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(addr, parity)) {
    if (global_timer_ns() - t0 > limit_ns) return;
  }
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    ns_gemm_kernel(const __grid_constant__ NsGemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* tiles = smem;
  uint8_t* epibuf = smem + kStages * kStageBytes;  // kEpiWarps x kEpiBufBytes, 1 KB aligned
  uint64_t* full = reinterpret_cast<uint64_t*>(epibuf + kEpiWarps * kEpiBufBytes);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* done = tempty + 2;
  uint64_t* epibar = done + 1;  // kEpiWarps x kEpiBufs
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(epibar + kEpiWarps * kEpiBufs);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint32_t* pubcnt = tmem_slot + 2;  // kPubSlots: epilogue warps that stored a tile, per slot

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint64_t limit = p.wait_limit_ns;
  const uint32_t rank = cluster_ctarank();  // 0: pair leader, issues the MMAs
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int npairs = static_cast<int>(gridDim.x >> 1);
  const int ntiles = p.ns_steps * tiles_per_step(p);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);   // the leader's: one arrival + both CTAs' bytes
      mbar_init(&empty[s], 1);  // one multicast commit from the leader's MMAs
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * kEpiWarps);  // the leader's: both CTAs' epilogue warps
    }
    mbar_init(done, 1);
    for (int w = 0; w < kEpiWarps * kEpiBufs; ++w) mbar_init(&epibar[w], 1);
    *abort_flag = 0;
    for (int i = 0; i < kPubSlots; ++i) pubcnt[i] = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    for (int b = 0; b < p.nbanks; ++b)
      for (int k = 0; k < kMaxMaps; ++k) tma_prefetch_map(&p.maps[b][k]);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the other CTA's barriers are initialised before any remote signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      const uint32_t full_leader = mapa_shared(smem_u32(full), 0);
      int stage = 0;
      uint32_t phase = 0;
      int issued_parity[kStages];
      for (int s = 0; s < kStages; ++s) issued_parity[s] = -1;
      bool ok = true;
      bool first = true;
      for (int tile = pair; ok && tile < ntiles; tile += npairs) {
        const Tile T = decode_tile(p, tile);
        if (T.phase == kReduce) continue;  // no MMA: the epilogue warps sum partials
        // the operands of this tile are final once the phase it reads is done
        if (!wait_dependency(T.dep_cnt, T.dep_target, abort_flag, p.status, limit)) {
          ok = false;
          break;
        }
        for (int kb = 0; kb < T.nkb; ++kb) {
          if (!mbar_wait_cluster(&empty[stage], phase ^ 1u, abort_flag, p.status, limit)) {
            ok = false;
            break;
          }
          const bool withhold = first && p.fault == 1 && blockIdx.x == 0;
          first = false;
          if (!withhold) {
            uint8_t* st = tiles + stage * kStageBytes;
            const uint32_t bar = full_leader + 8u * static_cast<uint32_t>(stage);
            // a diagonal block's right operand is the left one: not loaded
            if (rank == 0)
              mbar_arrive_expect_tx(&full[stage], T.same_ab ? 2 * kATileBytes : 2 * kStageBytes);
            const int k0 = (T.kb0 + kb) * kBK;
            const bool at = below_diagonal(T.a_sym, T.m0, k0);
            const bool bt = below_diagonal(T.b_sym, T.n0, k0);
            const BankPlan& bp = p.bank[T.bank];
            {
              const int slot = at ? T.a_tmap : T.a_map, mn = at ? 1 : T.a_mn;
              const int row = T.m0 + kBM * static_cast<int>(rank);
              const bool in_map = operand_in_bounds(p, bp, slot, mn, T.a_base, row, k0);
              load_operand(st, &p.maps[T.bank][slot], bar, mn, in_map ? T.a_base : 0, in_map ? row : 0,
                           in_map ? k0 : 0);
            }
            if (!T.same_ab) {
              const int slot = bt ? T.b_tmap : T.b_map, mn = bt ? 1 : T.b_mn;
              const int row = T.n0 + (kBN / 2) * static_cast<int>(rank);
              const bool in_map = operand_in_bounds(p, bp, slot, mn, T.b_base, row, k0);
              load_operand(st + kATileBytes, &p.maps[T.bank][slot], bar, mn, in_map ? T.b_base : 0,
                           in_map ? row : 0, in_map ? k0 : 0);
            }
            issued_parity[stage] = static_cast<int>(phase);
          }
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      }
      // the leader's full barriers count both CTAs' bytes: drain them there
      if (rank == 0)
        for (int s = 0; s < kStages; ++s)
          if (issued_parity[s] >= 0) drain_wait(&full[s], static_cast<uint32_t>(issued_parity[s]), limit);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      if (rank == 0) {
        // -------------------------------------------------- MMA issuer (leader)
        int stage = 0;
        uint32_t phase = 0;
        int acc = 0;
        uint32_t acc_phase = 0;
        bool ok = true;
        for (int tile = pair; ok && tile < ntiles; tile += npairs) {
          const Tile T = decode_tile(p, tile);
          if (T.phase == kReduce) continue;
          if (!mbar_wait_cluster(&tempty[acc], acc_phase ^ 1u, abort_flag, p.status, limit)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kBN);
          for (int kb = 0; kb < T.nkb; ++kb) {
            if (!mbar_wait_cluster(&full[stage], phase, abort_flag, p.status, limit)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t a_addr = smem_u32(tiles + stage * kStageBytes);
            // on a diagonal block each CTA's half of the right operand (N rows
            // 128 * rank ..) is its own rows of the left operand
            const uint32_t b_addr = T.same_ab ? a_addr : a_addr + kATileBytes;
            // the producer's choice of orientation for this K block
            const int k0 = (T.kb0 + kb) * kBK;
            const int a_mn = below_diagonal(T.a_sym, T.m0, k0) ? 1 : T.a_mn;
            const int b_mn = below_diagonal(T.b_sym, T.n0, k0) ? 1 : T.b_mn;
            const uint32_t idesc = idesc_bf16(2 * kBM, kBN, a_mn, b_mn);
#pragma unroll
            for (int ks = 0; ks < kBK / 16; ++ks) {
              umma_bf16_pair(d_tmem, operand_desc(a_addr, a_mn, ks), operand_desc(b_addr, b_mn, ks),
                             idesc, (kb > 0 || ks > 0) ? 1u : 0u);
            }
            umma_commit_pair(&empty[stage]);  // frees this stage in both CTAs
            if (++stage == kStages) { stage = 0; phase ^= 1u; }
          }
          if (!ok) break;
          umma_commit_pair(&tfull[acc]);
          acc ^= 1;
          if (acc == 0) acc_phase ^= 1u;
        }
        // every MMA has finished (both CTAs learn it) before TMEM is released
        umma_commit_pair(done);
      }
      drain_wait(done, 0, limit);
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    // warp w may read TMEM lanes 32*(w%4)..+31 (this CTA's tile rows); warps
    // 2..5 take accumulator columns 0..127 and warps 6..9 columns 128..255.
    //
    // The accumulator is handed back to the MMA as soon as the last chunk's
    // TMEM load has landed in registers. A tile is published one tile late:
    // its stores complete while the next tile is worked on, and each warp
    // confirms it after that tile's chunk loop. Before this warp could wait
    // on a tile whose dependency is not yet met, the pending tile is
    // confirmed at once, so a pending publish never holds up a tile that
    // needs it (a CTA keeps a publish pending only while its next tile can
    // run, and that tile finishes).
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    const int ew = warp - 2;
    const int irank = static_cast<int>(rank);
    EpiRing e{epibuf + ew * kEpiBufBytes, &epibar[ew * kEpiBufs], 0u, 0u, 0u};
    const uint32_t tempty_leader = mapa_shared(smem_u32(tempty), 0);
    constexpr int kChunks = 128 / kEpiCols;  // chunks per warp per tile
    static_assert(kEpiBufs <= kChunks, "the loads of one tile fill the ring");
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    int* pend_cnt = nullptr;   // lane 0: the tile whose publish is pending
    uint32_t pend_slot = 0;
    uint32_t seq = 0;          // MMA tiles handled by this warp
    for (int tile = pair; ok && tile < ntiles; tile += npairs) {
      const Tile T = decode_tile(p, tile);
      const BankPlan& bp = p.bank[T.bank];
      if (T.phase == kReduce) {  // no accumulator: sum the split partials
        // the Reduce needs every ring buffer free and waits on its dependency
        if (lane == 0) {
          bulk_wait_all();
          if (pend_cnt) {
            confirm_tile(&pubcnt[pend_slot], pend_cnt);
            pend_cnt = nullptr;
          }
          if (!wait_dependency(T.dep_cnt, T.dep_target, abort_flag, p.status, limit)) ok = false;
        }
        if (!__all_sync(0xffffffffu, ok)) break;
        if (!epi_reduce(p, e, T, bp, lane, irank, q, half, abort_flag)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          bulk_wait_all();
          fence_proxy_async_global();
          red_release_gpu_add(T.done_cnt, 1);
        }
        __syncwarp();
        continue;
      }
      const bool split = T.phase == kGram && bp.ksplit > 1;
      const int prow = (T.mat * bp.tiles_sym + T.sym_t) * bp.ksplit * kTile + T.split * kTile +
                       kBM * irank + 32 * q;
      const int r0 = T.m0 + kBM * irank + 32 * q;  // first row of this warp
      const int cw = T.n0 + half * 128;            // first column of this warp
      const bool loads = epi_has_loads(T);
      if (lane == 0) {
        // one acquire of the dependency counter serves both checks below
        const bool ready = !(pend_cnt || loads) || dependency_met(T);
        // a pending publish must not hold up this tile: confirm it first
        // whenever this tile's dependency is not yet met
        if (pend_cnt && !ready) {
          bulk_wait_all();
          confirm_tile(&pubcnt[pend_slot], pend_cnt);
          pend_cnt = nullptr;
        }
        if (loads) {
          // the epilogue's own loads read the same finished phase as the MMAs;
          // the first kEpiBufs chunks are requested now, while the MMAs run
          if (!ready && !wait_dependency(T.dep_cnt, T.dep_target, abort_flag, p.status, limit)) {
            ok = false;
          } else {
            fence_proxy_async_global();
            bulk_wait_read<0>();  // the previous tile's buffers have been read out
            for (int j = 0; j < kEpiBufs; ++j) epi_issue_chunk(p, e, T, irank, q, half, j, e.chunk + j);
          }
        }
      }
      if (!__all_sync(0xffffffffu, ok)) break;
      // the tcgen05.ld below is warp-collective: leave only if the whole warp does
      const bool got = mbar_wait_cluster(&tfull[acc], acc_phase, abort_flag, p.status, limit);
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(32 * q) << 16) +
                          static_cast<uint32_t>(acc * kBN + half * 128);
#pragma unroll 1
      for (int j = 0; j < kChunks; ++j) {
        const uint32_t k = e.chunk;
        const int c0 = cw + j * kEpiCols;
        if (lane == 0 && !loads) bulk_wait_read<kEpiBufs - 1>();  // buffer of chunk k: its store has read it
        __syncwarp();
        uint32_t r[32];
        tmem_ld32(tb + j * kEpiCols, r);
        if (loads && !epi_wait_load(p, e, k, abort_flag)) {
          tmem_ld_wait();
          ok = false;
          break;
        }
        tmem_ld_wait();
        if (j == kChunks - 1) {
          // every accumulator column of this warp is in registers: hand the
          // accumulator back. The arrive has the default (CTA-scope release)
          // semantics: a cluster-scope release measured ~14 % of the
          // epilogue's time per tile, and the TMEM reads it orders have
          // completed (tcgen05.wait::ld) before it. Lane 1 arrives; lane 0
          // issues the bulk stores.
          tc_fence_before();
          __syncwarp();
          if (lane == 1) mbar_arrive_cluster_cta(tempty_leader + 8u * static_cast<uint32_t>(acc));
        }
        uint8_t* buf = ring_buf(e, k);
        if (split) {
          epi_partial(p, T, buf, lane, prow, half * 128 + j * kEpiCols, r);
        } else {
          if (T.phase == kApply)
            epi_apply(T, bp, buf, lane, r);
          else
            epi_sym(T, bp, buf, lane, r);
          epi_store(p, T, bp, buf, r0, c0, lane);
        }
        if (loads && j + kEpiBufs < kChunks) {
          // chunk j's buffer takes chunk j + kEpiBufs once its store has read it
          __syncwarp();
          if (lane == 0) {
            bulk_wait_read<0>();
            epi_issue_chunk(p, e, T, irank, q, half, j + kEpiBufs, k + kEpiBufs);
          }
        }
        e.chunk = k + 1;
      }
      if (!ok) break;
      __syncwarp();
      if (lane == 0) {
        // the previous tile's stores are the groups before this tile's kChunks
        if (pend_cnt) {
          bulk_wait<kChunks>();
          confirm_tile(&pubcnt[pend_slot], pend_cnt);
        }
        pend_cnt = T.done_cnt;
        pend_slot = seq % kPubSlots;
      }
      ++seq;
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    if (lane == 0) {
      bulk_wait_all();  // every bulk store of this warp has completed
      if (ok && pend_cnt) confirm_tile(&pubcnt[pend_slot], pend_cnt);
      // after an error, loads may still be in flight: let them land before
      // the CTA's shared memory is released
      for (int i = 0; i < kEpiBufs; ++i)
        if (e.inflight & (1u << i)) drain_wait(&e.bar[i], (e.parity >> i) & 1u, limit);
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no MMA of the pair and no remote signal is still in flight
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

// One-time set-up on the current device: the kernel's shared-memory size and
// the number of CTA pairs that can be resident at once. The chain's tiles
// wait on tiles that other pairs own, so every pair of the grid must be
// resident together; the grid never exceeds what the occupancy calculator
// reports for this kernel's cluster and shared-memory configuration (on an
// otherwise idle device: one pair per TPC). Kernels of other streams that hold
// SMs only delay the pairs that cannot start yet; chains on several streams
// of one device serialise the same way.
cudaError_t ns_gemm_prepare(int* max_pairs) {
  cudaError_t e = cudaFuncSetAttribute(ns_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kGemmSmemBytes);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (sms / 2), 1, 1);
  cfg.blockDim = dim3(kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = kGemmSmemBytes;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int clusters = 0;
  if ((e = cudaOccupancyMaxActiveClusters(&clusters, ns_gemm_kernel, &cfg)) != cudaSuccess) return e;
  if (clusters < 1) return cudaErrorInvalidConfiguration;
  *max_pairs = clusters < sms / 2 ? clusters : sms / 2;
  return cudaSuccess;
}

cudaError_t launch_ns_gemm(const NsGemmParams& p, int max_pairs, cudaStream_t s) {
  const int tiles = p.ns_steps * tiles_per_step(p);
  int pairs = max_pairs;
  if (tiles < pairs) pairs = tiles;
  if (pairs < 1) pairs = 1;
  ns_gemm_kernel<<<2 * pairs, kGemmThreads, kGemmSmemBytes, s>>>(p);
  return cudaGetLastError();
}

}  // namespace muon
