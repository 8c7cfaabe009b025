// Periodic radius graph -> destination-sorted CSR, then per-edge distance and
// Wigner-D rows.
//
// Graph: "MALOQ: Massively Accelerated Learning of Operators for Quantum
// Transport", Section I and Table II (atoms within a cutoff radius, periodic
// cells); incoming-edge ownership from the review page of "Distributed
// Equivariant Graph Neural Networks for Large-Scale Electronic Structure
// Prediction", "What carries the argument".  Wigner-D: MALOQ Section III-C1 and
// Fig. 3 (rotate every edge to one axis, D^l for every degree, computed once
// per structure).  The D^l come from the 3x3 frame by the recursion of Ivanic
// and Ruedenberg (J. Phys. Chem. 100, 6342 (1996); erratum 102, 9099 (1998)),
// which builds the real-harmonic rotation of degree l from that of degree l-1
// and the l = 1 block; it needs no angles, only the rotation matrix.
//
// Kernels, in launch order:
//   cell_assign   atom -> cell, cell occupancy counts            (HBM: 24 B/atom)
//   scan          exclusive scan of counts (one CTA)
//   cell_fill     cell -> atom lists
//   nbr_count     per destination atom: candidates passing the exact test
//   scan          -> row_ptr
//   nbr_fill      per destination atom: rank-sort passing (s, shift) keys into
//                 the CSR segment (no global sort)            (HBM: 7 B/edge)
//   wigner        per edge: fp64 r_e, fp32 distance, frame and D^l rows
//                                                  (HBM: 4 + 4*wfl B/edge written)
#include <math.h>
#include <stdio.h>

#include "common.cuh"

namespace {

constexpr int kMaxSegment = 4096;   // incoming edges per atom (fill kernel's shared keys)
constexpr int kFillThreads = 256;

struct CellGrid {
  int brute;          // 1: every atom x every shift in [-S, S]^3
  int nc[3];          // cells per dimension (cell mode)
  double cw[3];       // cell widths (cell mode)
  int S[3];           // shift half-ranges (brute mode)
  double box[3];
  double rcut2;
};

// The exact inclusion test (separately rounded fp64 operations, fixed order).
__device__ __forceinline__ bool edge_test(const double* __restrict__ pos, int s, int d, int sx,
                                          int sy, int sz, const CellGrid& G) {
  double rx = __dsub_rn(__dadd_rn(pos[3 * s + 0], __dmul_rn((double)sx, G.box[0])), pos[3 * d + 0]);
  double ry = __dsub_rn(__dadd_rn(pos[3 * s + 1], __dmul_rn((double)sy, G.box[1])), pos[3 * d + 1]);
  double rz = __dsub_rn(__dadd_rn(pos[3 * s + 2], __dmul_rn((double)sz, G.box[2])), pos[3 * d + 2]);
  double d2 = __dadd_rn(__dadd_rn(__dmul_rn(rx, rx), __dmul_rn(ry, ry)), __dmul_rn(rz, rz));
  if (!(d2 < G.rcut2)) return false;
  return !(s == d && sx == 0 && sy == 0 && sz == 0);
}

__global__ void cell_assign_kernel(const double* __restrict__ pos, const int32_t* __restrict__ species,
                                   int n, CellGrid G, int32_t* __restrict__ atom_cell,
                                   int32_t* __restrict__ cell_count, int32_t* status) {
  int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  int c[3];
  bool bad = species[i] < 0;
  for (int k = 0; k < 3; ++k) {
    double x = pos[3 * i + k];
    if (!(x >= 0.0 && x < G.box[k])) bad = true;   // also catches NaN
    int ck = 0;
    if (!G.brute) {
      double q = x / G.cw[k];
      ck = (q >= 0.0) ? (int)q : 0;
      if (ck >= G.nc[k]) ck = G.nc[k] - 1;
    }
    c[k] = ck;
  }
  if (bad) egnn_flag(status, EGNN_DEV_BAD_POSITION);
  int lin = G.brute ? 0 : (c[0] * G.nc[1] + c[1]) * G.nc[2] + c[2];
  atom_cell[i] = lin;
  atomicAdd(cell_count + lin, 1);
}

// Exclusive scan of n int32 counts by one CTA; out[n] = total.  Total > INT32_MAX
// flags EGNN_DEV_EDGE_OVERFLOW and writes INT32_MAX.
__global__ void scan_kernel(const int32_t* __restrict__ in, int32_t* __restrict__ out, int n,
                            int32_t* status) {
  __shared__ long long part[1024];
  int t = threadIdx.x, T = blockDim.x;
  int per = (n + T - 1) / T;
  int b = t * per, e = min(n, b + per);
  long long s = 0;
  for (int i = b; i < e; ++i) s += in[i];
  part[t] = s;
  __syncthreads();
  for (int off = 1; off < T; off <<= 1) {
    long long v = (t >= off) ? part[t - off] : 0;
    __syncthreads();
    part[t] += v;
    __syncthreads();
  }
  long long run = (t == 0) ? 0 : part[t - 1];
  for (int i = b; i < e; ++i) {
    out[i] = (int32_t)(run > 0x7fffffffLL ? 0x7fffffffLL : run);
    run += in[i];
  }
  if (t == T - 1) {
    long long tot = part[T - 1];
    if (tot > 0x7fffffffLL) {
      egnn_flag(status, EGNN_DEV_EDGE_OVERFLOW);
      tot = 0x7fffffffLL;
    }
    out[n] = (int32_t)tot;
  }
}

__global__ void cell_fill_kernel(const int32_t* __restrict__ atom_cell, int n,
                                 const int32_t* __restrict__ cell_start, int32_t* __restrict__ cell_fill,
                                 int32_t* __restrict__ cell_atoms) {
  int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  int c = atom_cell[i];
  int slot = atomicAdd(cell_fill + c, 1);
  cell_atoms[cell_start[c] + slot] = i;
}

// Visit every candidate (s, shift) of destination d; f(s, sx, sy, sz) is called by
// the thread `lane` of `nl` cooperating threads for its share of candidates.
template <typename F>
__device__ __forceinline__ void for_candidates(int d, int n, const CellGrid& G,
                                               const int32_t* __restrict__ atom_cell,
                                               const int32_t* __restrict__ cell_start,
                                               const int32_t* __restrict__ cell_atoms, int lane,
                                               int nl, F&& f) {
  if (G.brute) {
    int ns0 = 2 * G.S[0] + 1, ns1 = 2 * G.S[1] + 1, ns2 = 2 * G.S[2] + 1;
    long long total = (long long)n * ns0 * ns1 * ns2;
    for (long long q = lane; q < total; q += nl) {
      int s = (int)(q / (ns0 * ns1 * ns2));
      int r = (int)(q - (long long)s * ns0 * ns1 * ns2);
      int sx = r / (ns1 * ns2) - G.S[0];
      int sy = (r / ns2) % ns1 - G.S[1];
      int sz = r % ns2 - G.S[2];
      f(s, sx, sy, sz);
    }
    return;
  }
  int lin = atom_cell[d];
  int cz = lin % G.nc[2];
  int cy = (lin / G.nc[2]) % G.nc[1];
  int cx = lin / (G.nc[2] * G.nc[1]);
  for (int o = 0; o < 27; ++o) {
    int t[3] = {cx + o / 9 - 1, cy + (o / 3) % 3 - 1, cz + o % 3 - 1};
    int sh[3], w[3];
    for (int k = 0; k < 3; ++k) {
      sh[k] = (t[k] < 0) ? -1 : (t[k] >= G.nc[k] ? 1 : 0);
      w[k] = t[k] - sh[k] * G.nc[k];
    }
    int c = (w[0] * G.nc[1] + w[1]) * G.nc[2] + w[2];
    int b = cell_start[c], e = cell_start[c + 1];
    for (int q = b + lane; q < e; q += nl) f(cell_atoms[q], sh[0], sh[1], sh[2]);
  }
}

// One warp per destination atom.
__global__ void nbr_count_kernel(const double* __restrict__ pos, int n, CellGrid G,
                                 const int32_t* __restrict__ atom_cell,
                                 const int32_t* __restrict__ cell_start,
                                 const int32_t* __restrict__ cell_atoms, int32_t* __restrict__ counts,
                                 int32_t* status) {
  int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  int lane = threadIdx.x & 31;
  if (warp >= n) return;
  int d = warp;
  int cnt = 0;
  for_candidates(d, n, G, atom_cell, cell_start, cell_atoms, lane, 32,
                 [&](int s, int sx, int sy, int sz) { cnt += edge_test(pos, s, d, sx, sy, sz, G); });
  for (int off = 16; off; off >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
  if (lane == 0) {
    if (cnt > kMaxSegment) {
      egnn_flag(status, EGNN_DEV_SEGMENT_TOO_LARGE);
      cnt = kMaxSegment;
    }
    counts[d] = cnt;
  }
}

// One CTA per destination atom: collect passing keys, then place each by rank.
__global__ void __launch_bounds__(kFillThreads) nbr_fill_kernel(
    const double* __restrict__ pos, int n, CellGrid G, const int32_t* __restrict__ atom_cell,
    const int32_t* __restrict__ cell_start, const int32_t* __restrict__ cell_atoms,
    const int32_t* __restrict__ row_ptr, int32_t* __restrict__ src, int8_t* __restrict__ shift,
    long long capacity, int32_t* status) {
  __shared__ long long keys[kMaxSegment];
  __shared__ int nk;
  int d = blockIdx.x;
  if (threadIdx.x == 0) nk = 0;
  __syncthreads();
  int sr0 = G.brute ? G.S[0] : 1, sr1 = G.brute ? G.S[1] : 1, sr2 = G.brute ? G.S[2] : 1;
  int n0 = 2 * sr0 + 1, n1 = 2 * sr1 + 1, n2 = 2 * sr2 + 1;
  long long nsh = (long long)n0 * n1 * n2;
  for_candidates(d, n, G, atom_cell, cell_start, cell_atoms, threadIdx.x, blockDim.x,
                 [&](int s, int sx, int sy, int sz) {
                   if (edge_test(pos, s, d, sx, sy, sz, G)) {
                     int slot = atomicAdd(&nk, 1);
                     long long code = ((long long)(sx + sr0) * n1 + (sy + sr1)) * n2 + (sz + sr2);
                     if (slot < kMaxSegment) keys[slot] = (long long)s * nsh + code;
                   }
                 });
  __syncthreads();
  int cnt = nk;
  int base = row_ptr[d];
  int expect = row_ptr[d + 1] - base;
  if (cnt != expect) {
    if (threadIdx.x == 0) egnn_flag(status, cnt > kMaxSegment ? EGNN_DEV_SEGMENT_TOO_LARGE
                                                              : EGNN_DEV_COUNT_MISMATCH);
    return;
  }
  for (int i = threadIdx.x; i < cnt; i += blockDim.x) {
    long long k = keys[i];
    int rank = 0;
    for (int j = 0; j < cnt; ++j) rank += keys[j] < k;
    long long pos_out = (long long)base + rank;
    if (pos_out >= capacity) {
      egnn_flag(status, EGNN_DEV_INDEX_RANGE);
      continue;
    }
    int s = (int)(k / nsh);
    int code = (int)(k - (long long)s * nsh);
    src[pos_out] = s;
    shift[3 * pos_out + 0] = (int8_t)(code / (n1 * n2) - sr0);
    shift[3 * pos_out + 1] = (int8_t)((code / n2) % n1 - sr1);
    shift[3 * pos_out + 2] = (int8_t)(code % n2 - sr2);
  }
}

constexpr int kLmaxW = 6;
constexpr int kDim = 2 * kLmaxW + 1;

// One thread per edge.  fp64 edge vector and frame, fp32 recursion.
__global__ void __launch_bounds__(128) wigner_kernel(
    const double* __restrict__ pos, int n, const int32_t* __restrict__ row_ptr,
    const int32_t* __restrict__ src, const int8_t* __restrict__ shift, long long n_edges, double bx,
    double by, double bz, int lmax, int mmax, int wfl, float* __restrict__ dist,
    float* __restrict__ wig, int32_t* status) {
  long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= n_edges) return;
  // destination atom: binary search of row_ptr
  int lo = 0, hi = n;
  while (hi - lo > 1) {
    int mid = (lo + hi) >> 1;
    if (row_ptr[mid] <= e) lo = mid; else hi = mid;
  }
  int d = lo, s = src[e];
  if (s < 0 || s >= n) {
    egnn_flag(status, EGNN_DEV_INDEX_RANGE);
    return;
  }
  double rx = __dsub_rn(__dadd_rn(pos[3 * s + 0], __dmul_rn((double)shift[3 * e + 0], bx)), pos[3 * d + 0]);
  double ry = __dsub_rn(__dadd_rn(pos[3 * s + 1], __dmul_rn((double)shift[3 * e + 1], by)), pos[3 * d + 1]);
  double rz = __dsub_rn(__dadd_rn(pos[3 * s + 2], __dmul_rn((double)shift[3 * e + 2], bz)), pos[3 * d + 2]);
  double r = sqrt(rx * rx + ry * ry + rz * rz);
  dist[e] = (float)r;
  double x = rx / r, y = ry / r, z = rz / r;
  double rho = sqrt(x * x + y * y);
  double ca = 1.0, sa = 0.0;
  if (rho > 0.0) { ca = x / rho; sa = y / rho; }
  // R = R_y(-beta) R_z(-alpha): rows (cb ca, cb sa, -sb), (-sa, ca, 0), (sb ca, sb sa, cb)
  double cb = z, sb = rho;
  double R[3][3] = {{cb * ca, cb * sa, -sb}, {-sa, ca, 0.0}, {sb * ca, sb * sa, cb}};
  // D^1 in the (y, z, x) component order: D1[i][j] = R[p(i)][p(j)], p = (1, 2, 0)
  const int p[3] = {1, 2, 0};
  float D1[3][3];
  for (int i = 0; i < 3; ++i)
    for (int j = 0; j < 3; ++j) D1[i][j] = (float)R[p[i]][p[j]];
  float Da[kDim * kDim], Db[kDim * kDim];   // previous / current degree
  float* wo = wig + e * (long long)wfl;
  wo[0] = 1.0f;
  if (lmax >= 1) {
    int m1 = mmax < 1 ? mmax : 1;
    int o = egnn_wig_off(1, mmax);
    for (int m = -m1; m <= m1; ++m)
      for (int j = 0; j < 3; ++j) wo[o + (m + m1) * 3 + j] = D1[m + 1][j];
    for (int i = 0; i < 9; ++i) Da[i] = D1[i / 3][i % 3];
  }
  float* prev = Da;
  float* cur = Db;
  for (int l = 2; l <= lmax; ++l) {
    int dp = 2 * l - 1, dc = 2 * l + 1;
    auto Pv = [&](int i, int a, int b) -> float {   // Ivanic-Ruedenberg P function
      float r1 = D1[i + 1][2], rm1 = D1[i + 1][0], r0 = D1[i + 1][1];
      if (b == l) return r1 * prev[(a + l - 1) * dp + (l - 1 + l - 1)] - rm1 * prev[(a + l - 1) * dp + 0];
      if (b == -l) return r1 * prev[(a + l - 1) * dp + 0] + rm1 * prev[(a + l - 1) * dp + (2 * l - 2)];
      return r0 * prev[(a + l - 1) * dp + (b + l - 1)];
    };
    for (int m = -l; m <= l; ++m) {
      int am = m < 0 ? -m : m;
      float dm0 = (m == 0) ? 1.f : 0.f;
      for (int nn = -l; nn <= l; ++nn) {
        float den = (nn > -l && nn < l) ? (float)((l + nn) * (l - nn)) : (float)(2 * l * (2 * l - 1));
        float u = sqrtf((float)((l + m) * (l - m)) / den);
        float v = 0.5f * sqrtf((1.f + dm0) * (float)((l + am - 1) * (l + am)) / den) * (1.f - 2.f * dm0);
        float wv = (float)((l - am - 1) * (l - am));
        float w = (m == 0 || wv <= 0.f) ? 0.f : -0.5f * sqrtf(wv / den);
        float val = 0.f;
        if (u != 0.f) val += u * Pv(0, m, nn);
        if (v != 0.f) {
          float V;
          if (m == 0) V = Pv(1, 1, nn) + Pv(-1, -1, nn);
          else if (m > 0) V = Pv(1, m - 1, nn) * (m == 1 ? 1.41421356237f : 1.f) - (m == 1 ? 0.f : Pv(-1, -m + 1, nn));
          else V = (m == -1 ? 0.f : Pv(1, m + 1, nn)) + Pv(-1, -m - 1, nn) * (m == -1 ? 1.41421356237f : 1.f);
          val += v * V;
        }
        if (w != 0.f) {
          float W;
          if (m > 0) W = Pv(1, m + 1, nn) + Pv(-1, -m - 1, nn);
          else W = Pv(1, m - 1, nn) - Pv(-1, -m + 1, nn);
          val += w * W;
        }
        cur[(m + l) * dc + (nn + l)] = val;
      }
    }
    int ml = l < mmax ? l : mmax;
    int o = egnn_wig_off(l, mmax);
    for (int m = -ml; m <= ml; ++m)
      for (int j = 0; j < dc; ++j) wo[o + (m + ml) * dc + j] = cur[(m + l) * dc + j];
    float* t = prev; prev = cur; cur = t;
  }
}

// ---- Wigner rows for lmax <= 4: the recursion unrolled per degree (registers), the
// rows of a CTA's 128 edges staged in shared memory and written out contiguously ----
__host__ __device__ constexpr int wig_floats_c(int lmax, int mmax) {
  int o = 0;
  for (int k = 0; k <= lmax; ++k) o += (2 * (k < mmax ? k : mmax) + 1) * (2 * k + 1);
  return o;
}

// Ivanic-Ruedenberg P function of degree l from the previous degree's matrix.
template <int l>
__device__ __forceinline__ float ir_P(const float (&D1)[3][3], const float* prev, int i, int a, int b) {
  constexpr int dp = 2 * l - 1;
  const float r1 = D1[i + 1][2], rm1 = D1[i + 1][0], r0 = D1[i + 1][1];
  if (b == l) return r1 * prev[(a + l - 1) * dp + (2 * l - 2)] - rm1 * prev[(a + l - 1) * dp];
  if (b == -l) return r1 * prev[(a + l - 1) * dp] + rm1 * prev[(a + l - 1) * dp + (2 * l - 2)];
  return r0 * prev[(a + l - 1) * dp + (b + l - 1)];
}

// D^l (row-major (2l+1)^2) from D^{l-1} and D^1, every index a compile-time constant.
template <int l>
__device__ __forceinline__ void ir_level(const float (&D1)[3][3], const float* prev, float* cur) {
  constexpr int dc = 2 * l + 1;
#pragma unroll
  for (int m = -l; m <= l; ++m) {
    const int am = m < 0 ? -m : m;
    const float dm0 = (m == 0) ? 1.f : 0.f;
#pragma unroll
    for (int nn = -l; nn <= l; ++nn) {
      const float den = (nn > -l && nn < l) ? (float)((l + nn) * (l - nn)) : (float)(2 * l * (2 * l - 1));
      const float u = sqrtf((float)((l + m) * (l - m)) / den);
      const float v = 0.5f * sqrtf((1.f + dm0) * (float)((l + am - 1) * (l + am)) / den) * (1.f - 2.f * dm0);
      const float wv = (float)((l - am - 1) * (l - am));
      const float w = (m == 0 || wv <= 0.f) ? 0.f : -0.5f * sqrtf(wv / den);
      float val = 0.f;
      if (l + m != 0 && l - m != 0) val += u * ir_P<l>(D1, prev, 0, m, nn);
      if (v != 0.f) {
        float V;
        if (m == 0) V = ir_P<l>(D1, prev, 1, 1, nn) + ir_P<l>(D1, prev, -1, -1, nn);
        else if (m > 0)
          V = ir_P<l>(D1, prev, 1, m - 1, nn) * (m == 1 ? 1.41421356237f : 1.f) -
              (m == 1 ? 0.f : ir_P<l>(D1, prev, -1, -m + 1, nn));
        else
          V = (m == -1 ? 0.f : ir_P<l>(D1, prev, 1, m + 1, nn)) +
              ir_P<l>(D1, prev, -1, -m - 1, nn) * (m == -1 ? 1.41421356237f : 1.f);
        val += v * V;
      }
      if (m != 0 && l - am - 1 > 0) {
        const float W = m > 0 ? ir_P<l>(D1, prev, 1, m + 1, nn) + ir_P<l>(D1, prev, -1, -m - 1, nn)
                              : ir_P<l>(D1, prev, 1, m - 1, nn) - ir_P<l>(D1, prev, -1, -m + 1, nn);
        val += w * W;
      }
      cur[(m + l) * dc + (nn + l)] = val;
    }
  }
}

// Kept rows |m| <= min(l, MM) of D^l into the edge's staged record.
template <int l, int MM>
__device__ __forceinline__ void keep_rows(const float* Dl, float* row) {
  constexpr int ml = l < MM ? l : MM, dc = 2 * l + 1, o = wig_floats_c(l - 1, MM);
#pragma unroll
  for (int m = -ml; m <= ml; ++m)
#pragma unroll
    for (int j = 0; j < dc; ++j) row[o + (m + ml) * dc + j] = Dl[(m + l) * dc + j];
}

// Edges per CTA of the tile kernel: 128 when their staged rows fit 48 KB, else 64.
template <int LM, int MM>
constexpr int wig_tile_edges() { return 128 * wig_floats_c(LM, MM) * 4 <= 48 * 1024 ? 128 : 64; }

template <int LM, int MM>
__global__ void __launch_bounds__(128) wigner_tile_kernel(
    const double* __restrict__ pos, int n, const int32_t* __restrict__ row_ptr,
    const int32_t* __restrict__ src, const int8_t* __restrict__ shift, long long n_edges, double bx,
    double by, double bz, float* __restrict__ dist, float* __restrict__ wig, int32_t* status) {
  constexpr int WFL = wig_floats_c(LM, MM), TE = wig_tile_edges<LM, MM>();
  __shared__ float rows[TE * WFL];
  __shared__ int ok[TE];
  const long long e0 = (long long)blockIdx.x * TE, e = e0 + threadIdx.x;
  const int nvalid = (int)(n_edges - e0 < TE ? n_edges - e0 : TE);
  float* row = rows + threadIdx.x * WFL;
  if (threadIdx.x < TE) ok[threadIdx.x] = 0;
  if (threadIdx.x < TE && e < n_edges) {
    int lo = 0, hi = n;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (row_ptr[mid] <= e) lo = mid; else hi = mid;
    }
    const int d = lo, s = src[e];
    if (s < 0 || s >= n) {
      egnn_flag(status, EGNN_DEV_INDEX_RANGE);
    } else {
      ok[threadIdx.x] = 1;
      const double rx = __dsub_rn(__dadd_rn(pos[3 * s + 0], __dmul_rn((double)shift[3 * e + 0], bx)), pos[3 * d + 0]);
      const double ry = __dsub_rn(__dadd_rn(pos[3 * s + 1], __dmul_rn((double)shift[3 * e + 1], by)), pos[3 * d + 1]);
      const double rz = __dsub_rn(__dadd_rn(pos[3 * s + 2], __dmul_rn((double)shift[3 * e + 2], bz)), pos[3 * d + 2]);
      const double r = sqrt(rx * rx + ry * ry + rz * rz);
      dist[e] = (float)r;
      const double x = rx / r, y = ry / r, z = rz / r;
      const double rho = sqrt(x * x + y * y);
      double ca = 1.0, sa = 0.0;
      if (rho > 0.0) {
        ca = x / rho;
        sa = y / rho;
      }
      // R = R_y(-beta) R_z(-alpha); D^1 in the (y, z, x) component order
      const double cb = z, sb = rho;
      const double R[3][3] = {{cb * ca, cb * sa, -sb}, {-sa, ca, 0.0}, {sb * ca, sb * sa, cb}};
      const int p[3] = {1, 2, 0};
      float D1[3][3];
#pragma unroll
      for (int i = 0; i < 3; ++i)
#pragma unroll
        for (int j = 0; j < 3; ++j) D1[i][j] = (float)R[p[i]][p[j]];
      row[0] = 1.0f;
      if constexpr (LM >= 1) {
        const float* D1f = &D1[0][0];
        keep_rows<1, MM>(D1f, row);
        if constexpr (LM >= 2) {
          float D2[25];
          ir_level<2>(D1, D1f, D2);
          keep_rows<2, MM>(D2, row);
          if constexpr (LM >= 3) {
            float D3[49];
            ir_level<3>(D1, D2, D3);
            keep_rows<3, MM>(D3, row);
            if constexpr (LM >= 4) {
              float D4[81];
              ir_level<4>(D1, D3, D4);
              keep_rows<4, MM>(D4, row);
            }
          }
        }
      }
    }
  }
  __syncthreads();
  // the CTA's edges are contiguous in the output: coalesced copy (edges with a bad
  // source index are left unwritten, as in the per-thread path)
  float* out = wig + e0 * WFL;
  for (int i = threadIdx.x; i < nvalid * WFL; i += blockDim.x)
    if (ok[i / WFL]) out[i] = rows[i];
}

}  // namespace

extern "C" int32_t egnn_wigner_floats(int32_t lmax, int32_t mmax) {
  if (lmax < 0 || mmax < 0) return 0;
  return egnn_wig_off(lmax + 1, mmax);
}

size_t egnn_graph_workspace_bytes(int32_t n_atoms) {
  size_t n = n_atoms > 0 ? (size_t)n_atoms : 0;
  size_t ncell = 2 * n + 64;
  size_t ints = n /*atom_cell*/ + (ncell + 1) /*cell_count*/ + (ncell + 1) /*cell_start*/ +
                ncell /*cell_fill*/ + n /*cell_atoms*/ + n /*counts*/ + 64;
  return ints * sizeof(int32_t) + 256;
}

// Wigner rows of every edge: the unrolled tile kernel up to lmax 4, the per-thread
// recursion beyond.
static cudaError_t launch_wigner(const double* pos, int n_atoms, const egnn_graph* g, long long E,
                                 const double box[3], int lmax, int mmax, cudaStream_t st) {
  const int blocks = (int)((E + 127) / 128);
  switch (mmax * 8 + lmax) {
#define EGNN_WT_CASE(LMv, MMv)                                                                         \
  case MMv * 8 + LMv:                                                                                 \
    wigner_tile_kernel<LMv, MMv><<<(int)((E + wig_tile_edges<LMv, MMv>() - 1) / wig_tile_edges<LMv, MMv>()), \
                                   wig_tile_edges<LMv, MMv>(), 0, st>>>(pos, n_atoms, g->row_ptr, g->src, g->shift, E, \
                                                         box[0], box[1], box[2], g->dist, g->wigner,  \
                                                         g->status);                                  \
    return cudaGetLastError();
    EGNN_WT_CASE(0, 0) EGNN_WT_CASE(1, 0) EGNN_WT_CASE(2, 0) EGNN_WT_CASE(3, 0) EGNN_WT_CASE(4, 0)
    EGNN_WT_CASE(1, 1) EGNN_WT_CASE(2, 1) EGNN_WT_CASE(3, 1) EGNN_WT_CASE(4, 1)
    EGNN_WT_CASE(2, 2) EGNN_WT_CASE(3, 2) EGNN_WT_CASE(4, 2)
#undef EGNN_WT_CASE
    default:
      break;
  }
  wigner_kernel<<<blocks, 128, 0, st>>>(pos, n_atoms, g->row_ptr, g->src, g->shift, E, box[0], box[1], box[2], lmax,
                                        mmax, egnn_wigner_floats(lmax, mmax), g->dist, g->wigner, g->status);
  return cudaGetLastError();
}

extern "C" egnn_status egnn_build_graph(const double* pos, const int32_t* species, int32_t n_atoms,
                                        const double box[3], double rcut, int32_t lmax, int32_t mmax,
                                        egnn_graph* g, void* workspace, size_t ws_bytes,
                                        void* cuda_stream) {
  if (!pos || !species || !box || !g || n_atoms < 1) return EGNN_ERR_INVALID_ARG;
  if (!(rcut > 0.0) || !g->row_ptr || !g->status) return EGNN_ERR_INVALID_ARG;
  if (lmax < 0 || lmax > kLmaxW || mmax < 0 || mmax > 2 || mmax > lmax) return EGNN_ERR_UNSUPPORTED;
  for (int k = 0; k < 3; ++k)
    if (!(box[k] > 0.0) || !(box[k] < 1e12)) return EGNN_ERR_INVALID_ARG;
  if (g->capacity < 0) return EGNN_ERR_INVALID_ARG;
  if (g->capacity > 0 && (!g->src || !g->shift || !g->dist || !g->wigner)) return EGNN_ERR_INVALID_ARG;
  size_t need = egnn_graph_workspace_bytes(n_atoms);
  if (!workspace || ws_bytes < need) return EGNN_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)cuda_stream;

  CellGrid G{};
  G.rcut2 = rcut * rcut;
  int nc[3];
  long long total = 1;
  for (int k = 0; k < 3; ++k) {
    G.box[k] = box[k];
    double q = box[k] / (rcut * 1.000001);
    nc[k] = q >= 1e6 ? 1000000 : (int)q;
  }
  // keep the cell count <= 2N + 64 (wider cells stay correct, only slower)
  while ((long long)nc[0] * nc[1] * nc[2] > 2LL * n_atoms + 64) {
    int k = (nc[0] >= nc[1] && nc[0] >= nc[2]) ? 0 : (nc[1] >= nc[2] ? 1 : 2);
    nc[k] = nc[k] * 3 / 4;
  }
  G.brute = (nc[0] < 3 || nc[1] < 3 || nc[2] < 3);
  for (int k = 0; k < 3; ++k) {
    G.nc[k] = G.brute ? 1 : nc[k];
    G.cw[k] = box[k] / G.nc[k];
    G.S[k] = (int)ceil(rcut / box[k]);
    if (G.S[k] > 100) return EGNN_ERR_UNSUPPORTED;
    total *= G.nc[k];
  }
  int ncell = (int)total;

  int32_t* w = (int32_t*)workspace;
  int32_t* atom_cell = w;                  w += n_atoms;
  int32_t* cell_count = w;                 w += ncell + 1;
  int32_t* cell_start = w;                 w += ncell + 1;
  int32_t* cell_fill = w;                  w += ncell;
  int32_t* cell_atoms = w;                 w += n_atoms;
  int32_t* counts = w;                     w += n_atoms;

  EGNN_CUDA_TRY(cudaMemsetAsync(g->status, 0, sizeof(int32_t), st));
  EGNN_CUDA_TRY(cudaMemsetAsync(cell_count, 0, sizeof(int32_t) * (ncell + 1), st));
  EGNN_CUDA_TRY(cudaMemsetAsync(cell_fill, 0, sizeof(int32_t) * ncell, st));
  int tb = 256;
  cell_assign_kernel<<<(n_atoms + tb - 1) / tb, tb, 0, st>>>(pos, species, n_atoms, G, atom_cell,
                                                              cell_count, g->status);
  scan_kernel<<<1, 1024, 0, st>>>(cell_count, cell_start, ncell, g->status);
  cell_fill_kernel<<<(n_atoms + tb - 1) / tb, tb, 0, st>>>(atom_cell, n_atoms, cell_start, cell_fill,
                                                            cell_atoms);
  nbr_count_kernel<<<(n_atoms * 32 + tb - 1) / tb, tb, 0, st>>>(pos, n_atoms, G, atom_cell, cell_start,
                                                                cell_atoms, counts, g->status);
  scan_kernel<<<1, 1024, 0, st>>>(counts, g->row_ptr, n_atoms, g->status);
  EGNN_CUDA_TRY(cudaGetLastError());
  int32_t E = 0, code = 0;
  EGNN_CUDA_TRY(cudaMemcpyAsync(&E, g->row_ptr + n_atoms, sizeof(int32_t), cudaMemcpyDeviceToHost, st));
  EGNN_CUDA_TRY(cudaMemcpyAsync(&code, g->status, sizeof(int32_t), cudaMemcpyDeviceToHost, st));
  EGNN_CUDA_TRY(cudaStreamSynchronize(st));
  g->n_atoms = n_atoms;
  g->lmax = lmax;
  g->mmax = mmax;
  g->n_edges = E;
  if (code != 0) return EGNN_ERR_DEVICE_CHECK;
  if ((int64_t)E > g->capacity) return EGNN_ERR_CAPACITY;
  if (E == 0) return EGNN_OK;
  nbr_fill_kernel<<<n_atoms, kFillThreads, 0, st>>>(pos, n_atoms, G, atom_cell, cell_start, cell_atoms,
                                                    g->row_ptr, g->src, g->shift, g->capacity, g->status);
  EGNN_CUDA_TRY(launch_wigner(pos, n_atoms, g, E, box, lmax, mmax, st));
  return EGNN_OK;
}

extern "C" egnn_status egnn_edge_geometry(const double* pos, const double box[3], egnn_graph* g,
                                          void* cuda_stream) {
  if (!pos || !box || !g || !g->row_ptr || !g->status || g->n_atoms < 1) return EGNN_ERR_INVALID_ARG;
  if (g->n_edges < 0 || g->n_edges > g->capacity || g->n_edges > 0x7fffffffLL) return EGNN_ERR_INVALID_ARG;
  if (g->n_edges > 0 && (!g->src || !g->shift || !g->dist || !g->wigner)) return EGNN_ERR_INVALID_ARG;
  if (g->lmax < 0 || g->lmax > kLmaxW || g->mmax < 0 || g->mmax > 2 || g->mmax > g->lmax)
    return EGNN_ERR_UNSUPPORTED;
  for (int k = 0; k < 3; ++k)
    if (!(box[k] > 0.0) || !(box[k] < 1e12)) return EGNN_ERR_INVALID_ARG;
  if (g->n_edges == 0) return EGNN_OK;
  cudaStream_t st = (cudaStream_t)cuda_stream;
  EGNN_CUDA_TRY(launch_wigner(pos, g->n_atoms, g, g->n_edges, box, g->lmax, g->mmax, st));
  return EGNN_OK;
}

// ---------------------------------------------------------------------------
// egnn_build_graph_noalloc: the same graph build for callers that cannot hand the
// library a device workspace.  Its scratch is a fixed array in this module's
// device memory; every GPU that loads the library holds one copy until exit.
// ---------------------------------------------------------------------------
#include <mutex>

namespace {

constexpr int32_t kNoAllocMaxAtoms = 131072;
// egnn_graph_workspace_bytes(n) needs 9n + 322 int32 words; round up generously.
constexpr size_t kNoAllocScratchWords = 9 * (size_t)kNoAllocMaxAtoms + 1024;

static __device__ __align__(256) int32_t g_noalloc_scratch[kNoAllocScratchWords];

std::mutex g_noalloc_mutex;
void* g_noalloc_addr[128] = {nullptr};

// Device address of g_noalloc_scratch on the current device.  The host-side name
// is only a stand-in, so the address is looked up once per device (with that
// device current) and cached.
egnn_status noalloc_scratch(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return EGNN_ERR_CUDA;
  if (dev < 0 || dev >= 128) return EGNN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_addr[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) return EGNN_ERR_CUDA;
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return EGNN_OK;
}

}  // namespace

extern "C" egnn_status egnn_build_graph_noalloc(const double* pos, const int32_t* species, int32_t n_atoms,
                                                const double box[3], double rcut, int32_t lmax, int32_t mmax,
                                                egnn_graph* g, void* cuda_stream) {
  if (n_atoms > kNoAllocMaxAtoms) return EGNN_ERR_UNSUPPORTED;
  if (!pos || !species || !box || !g || n_atoms < 1) return EGNN_ERR_INVALID_ARG;
  size_t need = egnn_graph_workspace_bytes(n_atoms);
  if (need > sizeof(int32_t) * kNoAllocScratchWords) return EGNN_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  egnn_status s = noalloc_scratch(&scratch);
  if (s != EGNN_OK) return s;
  return egnn_build_graph(pos, species, n_atoms, box, rcut, lmax, mmax, g, scratch,
                          sizeof(int32_t) * kNoAllocScratchWords, cuda_stream);
}
