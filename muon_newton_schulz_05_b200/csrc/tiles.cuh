// One tile of the Newton-Schulz chain: which product, which output block,
// which operands, and which counter it waits on. Shared by the chain kernel
// and the host-side description of its work list (muon_chain_plan).
#pragma once
#include "plan.cuh"

namespace muon {

struct Tile {
  int bank, mat, m0, n0, nkb;
  int kb0;                    // first 64-deep K block (split Gram tiles)
  int sym_t, split, sub;      // symmetric tile index, K split, reduce sub-tile
  int phase, iter, cur;       // Phase, Newton-Schulz step, hi buffer holding X_iter
  float a, b, c;              // this step's coefficients
  int a_map, a_mn, a_base;
  int b_map, b_mn, b_base;
  int a_sym, b_sym;           // operand is A or B: blocks below the diagonal read transposed
  int a_tmap, b_tmap;         // the MN-major map for those blocks
  int same_ab;                // diagonal block of a symmetric product: each CTA's half of
                              // the right operand is its own rows of the left operand
  int* done_cnt;              // counter this tile's epilogue advances
  const int* dep_cnt;         // counter of the phase this tile reads
  int dep_target;             // value dep_cnt must reach first (0: nothing to wait for)
};

// Upper 256 x 256 tiles (diagonal included) of a symmetric product with nb
// block rows: block row i holds block columns i .. nb-1.
__host__ __device__ __forceinline__ void sym_tile(int t, int nb, int& i, int& j) {
  int ii = 0;
  while (t >= nb - ii) {
    t -= nb - ii;
    ++ii;
  }
  i = ii;
  j = ii + t;
}


__host__ __device__ __forceinline__ Tile decode_tile(const NsGemmParams& p, int tile) {
  Tile T;
  const int G = p.gram_begin[p.nbanks], Rd = p.red_begin[p.nbanks], S = p.sym_begin[p.nbanks];
  const int per_iter = tiles_per_step(p);
  T.iter = fdiv(tile, p.fd_step);
  int r = tile - T.iter * per_iter;
  const int* begin;
  if (r < G) {
    T.phase = kGram;
    begin = p.gram_begin;
  } else if (r < G + Rd) {
    T.phase = kReduce;
    r -= G;
    begin = p.red_begin;
  } else if (r < G + Rd + S) {
    T.phase = kPoly;
    r -= G + Rd;
    begin = p.sym_begin;
  } else {
    T.phase = kApply;
    r -= G + Rd + S;
    begin = p.apply_begin;
  }
  int b = 0;
  while (b + 1 < p.nbanks && r >= begin[b + 1]) ++b;
  const BankPlan& bp = p.bank[b];
  const int local = r - begin[b];
  T.bank = b;
  T.cur = T.iter & 1;
  T.a = p.coef[3 * T.iter];
  T.b = p.coef[3 * T.iter + 1];
  T.c = p.coef[3 * T.iter + 2];
  T.kb0 = 0;
  T.split = 0;
  T.sub = 0;
  T.sym_t = 0;
  T.a_sym = T.b_sym = 0;
  T.a_tmap = T.b_tmap = 0;
  T.same_ab = 0;
  if (T.phase == kApply) {
    T.mat = fdiv(local, bp.fd_apply);
    const int t = local - T.mat * bp.tiles_apply;
    const int nbn = bp.Cp / kTile;
    const int mrow = fdiv(t, bp.fd_nbn);
    T.m0 = mrow * kTile;
    T.n0 = (t - mrow * nbn) * kTile;
  } else {
    int t;
    if (T.phase == kGram) {
      const int per = bp.tiles_sym * bp.ksplit;
      T.mat = fdiv(local, bp.fd_gram);
      const int t2 = local - T.mat * per;
      t = fdiv(t2, bp.fd_ksplit);
      T.split = t2 - t * bp.ksplit;
    } else if (T.phase == kReduce) {
      T.mat = fdiv(local, bp.fd_red);
      const int t3 = local - T.mat * bp.tiles_red;
      t = t3 / kRedSub;
      T.sub = t3 - t * kRedSub;
    } else {
      T.mat = fdiv(local, bp.fd_sym);
      t = local - T.mat * bp.tiles_sym;
    }
    T.sym_t = t;
    int i, j;
    sym_tile(t, bp.rp / kTile, i, j);
    T.m0 = i * kTile;
    T.n0 = j * kTile;
    // Gram and Poly read the same matrix on both sides (X X^T, A A); on a
    // diagonal block both sides are the same 256 rows, in the same
    // orientation for every K block
    T.same_ab = (T.phase != kReduce && i == j) ? 1 : 0;
  }
  // Gram(k) reads X_k (all of Apply(k-1)); Reduce(k) sums all of Gram(k)'s
  // partials; Poly(k) reads A (all of Reduce(k), or of Gram(k) when the bank
  // is not split); Apply(k) reads B (all of Poly(k)). Earlier phases are
  // implied by these.
  int* cnt = bp.counters + 4 * T.mat;
  T.done_cnt = cnt + T.phase;
  if (T.phase == kGram) {
    T.dep_cnt = cnt + kApply;
    T.dep_target = kTileParts * bp.tiles_apply * T.iter;
  } else if (T.phase == kReduce) {
    T.dep_cnt = cnt + kGram;
    T.dep_target = kTileParts * bp.tiles_sym * bp.ksplit * (T.iter + 1);
  } else if (T.phase == kPoly) {
    if (bp.ksplit > 1) {
      T.dep_cnt = cnt + kReduce;
      T.dep_target = kRedParts * bp.tiles_red * (T.iter + 1);
    } else {
      T.dep_cnt = cnt + kGram;
      T.dep_target = kTileParts * bp.tiles_sym * (T.iter + 1);
    }
  } else {
    T.dep_cnt = cnt + kPoly;
    T.dep_target = kTileParts * bp.tiles_sym * (T.iter + 1);
  }
  const int cur = T.cur;
  const int xbase = T.mat * bp.Rp;   // first row of this matrix in the iterate maps
  const int sbase = T.mat * bp.rp;   // first row of this matrix in the A / B maps
  if (T.phase == kGram) {
    if (!bp.tall) {  // D[m][n] = sum_k X[m][k] X[n][k]
      T.a_map = kHiK0 + cur; T.a_mn = 0; T.a_base = xbase;
      T.b_map = kHiK0 + cur; T.b_mn = 0; T.b_base = xbase;
      T.nkb = bp.Cp / kBK;
    } else {         // D[m][n] = sum_k Y[k][m] Y[k][n]
      T.a_map = kHiMN0 + cur; T.a_mn = 1; T.a_base = xbase;
      T.b_map = kHiMN0 + cur; T.b_mn = 1; T.b_base = xbase;
      T.nkb = bp.Rp / kBK;
    }
    if (bp.ksplit > 1) {  // this split's K blocks
      T.kb0 = T.split * bp.kc;
      T.nkb = min(bp.kc, T.nkb - T.kb0);
    }
  } else if (T.phase == kReduce) {
    T.nkb = 0;
    T.a_map = T.b_map = 0;
    T.a_mn = T.b_mn = 0;
    T.a_base = T.b_base = 0;
  } else if (T.phase == kPoly) {  // D[m][n] = sum_k A[m][k] A[n][k]
    T.a_map = kAK; T.a_mn = 0; T.a_base = sbase; T.a_sym = 1; T.a_tmap = kAMN;
    T.b_map = kAK; T.b_mn = 0; T.b_base = sbase; T.b_sym = 1; T.b_tmap = kAMN;
    T.nkb = bp.rp / kBK;
  } else {
    if (!bp.tall) {  // D[m][n] = sum_k B[m][k] X[k][n]
      T.a_map = kBK_; T.a_mn = 0; T.a_base = sbase; T.a_sym = 1; T.a_tmap = kBMN;
      T.b_map = kHiMN0 + cur; T.b_mn = 1; T.b_base = xbase;
      T.nkb = bp.Rp / kBK;
    } else {         // D[m][n] = sum_k Y[m][k] B[n][k]
      T.a_map = kHiK0 + cur; T.a_mn = 0; T.a_base = xbase;
      T.b_map = kBK_; T.b_mn = 0; T.b_base = sbase; T.b_sym = 1; T.b_tmap = kBMN;
      T.nkb = bp.Cp / kBK;
    }
  }
  return T;
}

}  // namespace muon
