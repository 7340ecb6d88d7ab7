// bcq_quantize.cu -- the offline multi-precision BCQ quantiser (bcq_quantize,
// and bcq_quantize_zp for offsets per precision).
//
// "AnyBCQ ..." (Paper-Notes page), "关键设计 / 渐进式精度扩展": at the base
// precision p_L the codes start greedy and are refined by alternating a
// least-squares fit of the scales with a nearest-code update; each expansion
// p -> p + 1 keeps B_1..B_p, appends B_{p+1} = sign(R_p) and refits every
// scale of alpha^(p+1) by least squares.  "训练策略": asymmetric, group 128,
// 20 refinement rounds.
//
// A quarter warp (8 lanes) quantises one 128-weight group (four groups per
// warp, so the per-group work every lane repeats -- Gram counts, the solve,
// candidate values -- is shared by four groups); lane j of a group holds
// columns j + 8 s, s = 0..15, so the ballot of plane bit i over slot s
// carries 8 columns of each of the warp's groups, and three byte permutes of
// four ballots give a canonical 32-column plane word.  Everything is fp64 (the weights are fp16,
// widened exactly).  Per step:
//   * the Gram matrix of the +-1 planes (and the all-ones column of z) is
//     integer-valued and comes exactly from popcounts of the plane words;
//   * right-hand sides are sums over the group's lanes (xor butterfly: every
//     lane ends with the same bits, since a + b == b + a), so every lane
//     solves the same system and holds the same scales without a broadcast;
//   * columns exactly dependent on the columns before them (a plane equal to
//     another, to its negation or to the all-ones column, or any exact linear
//     dependence) get scale 0; the normal equations of the kept columns are
//     solved by Cramer's rule with the exact integer adjugate;
//   * the code update gives every weight the code whose value
//     z + (((alpha_1 b_1) + alpha_2 b_2) + ...) is nearest, first code in
//     enumeration order on ties (code c: b_i = +1 where bit i of c is set).
// The greedy start peels b = sign(r), alpha = <b, r> / 128 off r = w - mean(w);
// sign(0) = +1.  z is fitted jointly with the base precision's scales and
// kept for the expansions (bcq_quantize_zp: refit with the scales at every
// expansion, giving z^(p) per precision).
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "bcq.h"

namespace bcq {
namespace {

constexpr int kQuantGroup = 128;
constexpr int kGroupLanes = 8;                        // lanes per group (quarter warp)
constexpr int kSlots = kQuantGroup / kGroupLanes;     // weights per lane
constexpr int kQuantWarps = 8;                        // warps per CTA (four groups each)
// kQuantMinCtas: two CTAs (16 warps, 64 groups) per SM, 128 registers a
// thread.  Measured on a 14336 x 4096 weight (p_L = 2 -> p_H = 4): 2.53 ms
// with four groups per warp, against 2.83 ms at one CTA per SM (230
// registers), 3.07 ms with two groups per warp and 3.77 ms with one (the
// per-group work each lane repeats is paid once per warp).
constexpr int kQuantMinCtas = 2;

struct QuantParams {
  const __half* w;       // fp16 [N][K]
  uint32_t* planes;      // uint32 [p_H][N][K/32]
  __half* alpha[4];      // alpha[q-1]: fp16 [N][G][q] (q = p_L..p_H)
  __half* z;             // fp16 [N][G] (shared offsets)
  __half* zq[4];         // per-precision offsets: zq[p-1] fp16 [N][G] (p = p_L..p_H)
  double* sse;           // fp64 [p_H - p_L + 1][N][G], or nullptr
  long long groups;      // N * G
  int N, K, G, rounds;
};

// Sum over the 8 lanes of this lane's group (xor butterfly within the group).
__device__ __forceinline__ double group_sum(double v) {
#pragma unroll
  for (int o = kGroupLanes / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Two group sums at once (lanes 0-3 of the group reduce a, lanes 4-7 reduce
// b, then both are broadcast within the group).  Only for sums that are
// exact in any order: sums of +-fp16 weights, whose partial sums are
// multiples of 2^-24 below 2^23.
__device__ __forceinline__ void group_sum2_exact(double a, double b, double& sa, double& sb) {
  const bool hi = (threadIdx.x & 4) != 0;
  double keep = hi ? b : a;
  keep += __shfl_xor_sync(0xffffffffu, hi ? a : b, 4);
#pragma unroll
  for (int o = 2; o > 0; o >>= 1) keep += __shfl_xor_sync(0xffffffffu, keep, o);
  const int base = threadIdx.x & 24;
  sa = __shfl_sync(0xffffffffu, keep, base);
  sb = __shfl_sync(0xffffffffu, keep, base + 4);
}

__device__ __forceinline__ double signed_val(bool plus, double a) { return plus ? a : -a; }

// x_a = (adj[a][0] r_0 + adj[a][1] r_1 + ...) / det: products and sums
// rounded one at a time, left to right (no contraction into fma).
template <int K, typename T>
__device__ __forceinline__ double cramer_row(const T (&adj)[K], const double (&r)[K],
                                             long long det) {
  double acc = __dmul_rn((double)adj[0], r[0]);
#pragma unroll
  for (int b = 1; b < K; ++b) acc = __dadd_rn(acc, __dmul_rn((double)adj[b], r[b]));
  return __ddiv_rn(acc, (double)det);
}

// Any M <= 5, any dependent columns: the kept columns (each independent of
// the kept columns before it) by symmetric fraction-free elimination on
// G / 2 -- a zero pivot of the positive semidefinite Schur complement means
// its whole row and column are zero, so skipping it keeps the elimination
// exact -- then the exact adjugate and determinant of the kept columns' Gram
// matrix by fraction-free Gauss-Jordan elimination of [G/2 | I] (left block
// det I, right block the adjugate; every division is exact; products in
// 128 bits), scaled back to G: adj(G) = 2^(k-1) adj(G/2), det(G) = 2^k det(G/2).
template <int M>
__device__ __forceinline__ void solve_general(const int (&G)[M][M], const double (&r)[M],
                                              double (&x)[M]) {
  // Local copies (static indexes only on the caller's arrays, so that they
  // stay in registers on the fast paths); dynamic indexes below touch only
  // these.
  long long S[M][M];
  int Gc[M][M];
  double rc[M], xs[M];
#pragma unroll
  for (int i = 0; i < M; ++i) {
    rc[i] = r[i];
    xs[i] = 0.0;
#pragma unroll
    for (int j = 0; j < M; ++j) {
      Gc[i][j] = G[i][j];
      S[i][j] = G[i][j] / 2;
    }
  }
  int idx[M];
  int k = 0;
  long long prev = 1;
#pragma unroll
  for (int c = 0; c < M; ++c) {
    if (S[c][c] == 0) continue;
    idx[k++] = c;
#pragma unroll
    for (int i = c + 1; i < M; ++i)
#pragma unroll
      for (int j = c + 1; j < M; ++j) S[i][j] = (S[c][c] * S[i][j] - S[i][c] * S[c][j]) / prev;
    prev = S[c][c];
  }
  long long A[M][2 * M];
  for (int a = 0; a < k; ++a)
    for (int b = 0; b < k; ++b) {
      A[a][b] = Gc[idx[a]][idx[b]] / 2;
      A[a][k + b] = a == b ? 1 : 0;
    }
  prev = 1;
  for (int c = 0; c < k; ++c) {
    const long long p = A[c][c];
    for (int i = 0; i < k; ++i) {
      if (i == c) continue;
      const long long f = A[i][c];
      for (int j = 0; j < 2 * k; ++j)
        A[i][j] = (long long)(((__int128)p * A[i][j] - (__int128)f * A[c][j]) / prev);
    }
    prev = p;
  }
  const long long det = prev * (1ll << k);
  const long long sc = 1ll << (k - 1);  // adj(G) = 2^(k-1) adj(G / 2)
  for (int a = 0; a < k; ++a) {
    double acc = __dmul_rn((double)(A[a][k] * sc), rc[idx[0]]);
    for (int b = 1; b < k; ++b) acc = __dadd_rn(acc, __dmul_rn((double)(A[a][k + b] * sc), rc[idx[b]]));
    xs[idx[a]] = __ddiv_rn(acc, (double)det);
  }
#pragma unroll
  for (int j = 0; j < M; ++j) x[j] = xs[j];
}

// Determinant of the 4x4 minor of a 5x5 integer matrix without row SR and
// column SC, by Laplace expansion over the 2x2 minors of its first two rows
// (s) and last two rows (c).  |G| <= 128: 2x2 minors below 2^15, the result
// below 2^33 (64-bit).
template <int SR, int SC>
__device__ __forceinline__ long long minor4(const int (&G)[5][5]) {
  int a[4][4];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) a[r][c] = G[r < SR ? r : r + 1][c < SC ? c : c + 1];
  const int s0 = a[0][0] * a[1][1] - a[1][0] * a[0][1], s1 = a[0][0] * a[1][2] - a[1][0] * a[0][2],
            s2 = a[0][0] * a[1][3] - a[1][0] * a[0][3], s3 = a[0][1] * a[1][2] - a[1][1] * a[0][2],
            s4 = a[0][1] * a[1][3] - a[1][1] * a[0][3], s5 = a[0][2] * a[1][3] - a[1][2] * a[0][3];
  const int c5 = a[2][2] * a[3][3] - a[3][2] * a[2][3], c4 = a[2][1] * a[3][3] - a[3][1] * a[2][3],
            c3 = a[2][1] * a[3][2] - a[3][1] * a[2][2], c2 = a[2][0] * a[3][3] - a[3][0] * a[2][3],
            c1 = a[2][0] * a[3][2] - a[3][0] * a[2][2], c0 = a[2][0] * a[3][1] - a[3][0] * a[2][1];
  return (long long)s0 * c5 - (long long)s1 * c4 + (long long)s2 * c3 + (long long)s3 * c2 -
         (long long)s4 * c1 + (long long)s5 * c0;
}

// Least squares on M columns with integer Gram matrix G and right-hand
// sides r, by Cramer's rule with the exact adjugate; columns dependent on
// earlier ones get 0.  Full-rank systems of 1 to 5 columns (every leading
// principal minor non-zero) take closed forms; the rest solve_general.
template <int M>
__device__ __forceinline__ void solve_exact(const int (&G)[M][M], const double (&r)[M],
                                            double (&x)[M]) {
  if constexpr (M == 1) {
    x[0] = __ddiv_rn(r[0], (double)G[0][0]);  // adj = [1]; G[0][0] = 128
    return;
  } else if constexpr (M == 2) {
    const int det = G[0][0] * G[1][1] - G[0][1] * G[1][0];
    if (det != 0) {
      const int a0[2] = {G[1][1], -G[0][1]}, a1[2] = {-G[1][0], G[0][0]};
      x[0] = cramer_row<2>(a0, r, det);
      x[1] = cramer_row<2>(a1, r, det);
      return;
    }
  } else if constexpr (M == 3) {
    const int g00 = G[0][0], g01 = G[0][1], g02 = G[0][2], g11 = G[1][1], g12 = G[1][2],
              g22 = G[2][2];
    // |G| <= 128: cofactors below 2^15, the determinant below 2^24
    const int c00 = g11 * g22 - g12 * g12, c01 = g02 * g12 - g01 * g22,
              c02 = g01 * g12 - g02 * g11, c11 = g00 * g22 - g02 * g02,
              c12 = g01 * g02 - g00 * g12, c22 = g00 * g11 - g01 * g01;
    const int det = g00 * c00 + g01 * c01 + g02 * c02;
    if (c22 != 0 && det != 0) {  // leading minors: g00 = 128, c22, det
      const int a0[3] = {c00, c01, c02}, a1[3] = {c01, c11, c12}, a2[3] = {c02, c12, c22};
      x[0] = cramer_row<3>(a0, r, det);
      x[1] = cramer_row<3>(a1, r, det);
      x[2] = cramer_row<3>(a2, r, det);
      return;
    }
  } else if constexpr (M == 4) {
    // Laplace expansion by the 2x2 minors of rows 0-1 (s) and rows 2-3 (c)
    // |G| <= 128: 2x2 minors below 2^15, adjugate entries (3x3 minors)
    // below 2^24, the determinant below 2^33 (64-bit)
    const int a00 = G[0][0], a01 = G[0][1], a02 = G[0][2], a03 = G[0][3];
    const int a11 = G[1][1], a12 = G[1][2], a13 = G[1][3];
    const int a22 = G[2][2], a23 = G[2][3], a33 = G[3][3];
    const int a10 = a01, a20 = a02, a21 = a12, a30 = a03, a31 = a13, a32 = a23;
    const int s0 = a00 * a11 - a10 * a01, s1 = a00 * a12 - a10 * a02,
              s2 = a00 * a13 - a10 * a03, s3 = a01 * a12 - a11 * a02,
              s4 = a01 * a13 - a11 * a03, s5 = a02 * a13 - a12 * a03;
    const int c5 = a22 * a33 - a32 * a23, c4 = a21 * a33 - a31 * a23,
              c3 = a21 * a32 - a31 * a22, c2 = a20 * a33 - a30 * a23,
              c1 = a20 * a32 - a30 * a22, c0 = a20 * a31 - a30 * a21;
    const long long det = (long long)s0 * c5 - (long long)s1 * c4 + (long long)s2 * c3 +
                          (long long)s3 * c2 - (long long)s4 * c1 + (long long)s5 * c0;
    const int b00 = a11 * c5 - a12 * c4 + a13 * c3, b01 = -a01 * c5 + a02 * c4 - a03 * c3,
              b02 = a31 * s5 - a32 * s4 + a33 * s3, b03 = -a21 * s5 + a22 * s4 - a23 * s3,
              b11 = a00 * c5 - a02 * c2 + a03 * c1, b12 = -a30 * s5 + a32 * s2 - a33 * s1,
              b13 = a20 * s5 - a22 * s2 + a23 * s1, b22 = a30 * s4 - a31 * s2 + a33 * s0,
              b23 = -a20 * s4 + a21 * s2 - a23 * s0, b33 = a20 * s3 - a21 * s1 + a22 * s0;
    if (s0 != 0 && b33 != 0 && det != 0) {  // leading minors: a00, s0, b33 (= 3x3), det
      const int r0[4] = {b00, b01, b02, b03}, r1[4] = {b01, b11, b12, b13},
                r2[4] = {b02, b12, b22, b23}, r3[4] = {b03, b13, b23, b33};
      x[0] = cramer_row<4>(r0, r, det);
      x[1] = cramer_row<4>(r1, r, det);
      x[2] = cramer_row<4>(r2, r, det);
      x[3] = cramer_row<4>(r3, r, det);
      return;
    }
  }
  else if constexpr (M == 5) {
    // adj[i][j] = (-1)^(i+j) det(G without row j, column i); G symmetric, so
    // adj is symmetric: 15 distinct 4x4 minors (below 2^33)
    long long A[5][5];
    A[0][0] = minor4<0, 0>(G);
    A[0][1] = -minor4<1, 0>(G);
    A[0][2] = minor4<2, 0>(G);
    A[0][3] = -minor4<3, 0>(G);
    A[0][4] = minor4<4, 0>(G);
    A[1][1] = minor4<1, 1>(G);
    A[1][2] = -minor4<2, 1>(G);
    A[1][3] = minor4<3, 1>(G);
    A[1][4] = -minor4<4, 1>(G);
    A[2][2] = minor4<2, 2>(G);
    A[2][3] = -minor4<3, 2>(G);
    A[2][4] = minor4<4, 2>(G);
    A[3][3] = minor4<3, 3>(G);
    A[3][4] = -minor4<4, 3>(G);
    A[4][4] = minor4<4, 4>(G);
#pragma unroll
    for (int i = 1; i < 5; ++i)
#pragma unroll
      for (int j = 0; j < i; ++j) A[i][j] = A[j][i];
    long long det = 0;  // expansion along row 0: sum_j G[0][j] adj[j][0]
#pragma unroll
    for (int j = 0; j < 5; ++j) det += (long long)G[0][j] * A[j][0];
    // leading minors: G[0][0] = 128, 2x2, 3x3, 4x4 (= adj[4][4]), det
    const long long d2 = (long long)G[0][0] * G[1][1] - (long long)G[0][1] * G[1][0];
    const long long d3 = (long long)G[0][0] * ((long long)G[1][1] * G[2][2] - (long long)G[1][2] * G[2][1]) -
                         (long long)G[0][1] * ((long long)G[1][0] * G[2][2] - (long long)G[1][2] * G[2][0]) +
                         (long long)G[0][2] * ((long long)G[1][0] * G[2][1] - (long long)G[1][1] * G[2][0]);
    if (d2 != 0 && d3 != 0 && A[4][4] != 0 && det != 0) {
#pragma unroll
      for (int a = 0; a < 5; ++a) x[a] = cramer_row<5>(A[a], r, det);
      return;
    }
  }
  if constexpr (M >= 2) solve_general<M>(G, r, x);
}

// Canonical words of plane i of this lane's group: word t = columns
// 32 t..32 t + 31 = slots 4t..4t + 3 (bytes 0..3), the group's byte of each
// ballot picked by byte permutes.
__device__ __forceinline__ void plane_word(const unsigned (&code)[kSlots], int i,
                                           uint32_t (&cw)[4]) {
  const uint32_t gq = (threadIdx.x >> 3) & 3u;
  const uint32_t sel = gq | ((gq + 4u) << 4);
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const uint32_t b0 = __ballot_sync(0xffffffffu, (code[4 * t] >> i) & 1u);
    const uint32_t b1 = __ballot_sync(0xffffffffu, (code[4 * t + 1] >> i) & 1u);
    const uint32_t b2 = __ballot_sync(0xffffffffu, (code[4 * t + 2] >> i) & 1u);
    const uint32_t b3 = __ballot_sync(0xffffffffu, (code[4 * t + 3] >> i) & 1u);
    cw[t] = __byte_perm(__byte_perm(b0, b1, sel), __byte_perm(b2, b3, sel), 0x5410u);
  }
}
template <int P>
__device__ __forceinline__ void plane_words(const unsigned (&code)[kSlots], uint32_t (&pw)[P][4]) {
#pragma unroll
  for (int i = 0; i < P; ++i) plane_word(code, i, pw[i]);
}

__device__ __forceinline__ int dot_pm1(const uint32_t (&a)[4], const uint32_t (&b)[4]) {
  return kQuantGroup - 2 * (__popc(a[0] ^ b[0]) + __popc(a[1] ^ b[1]) +
                            __popc(a[2] ^ b[2]) + __popc(a[3] ^ b[3]));
}
__device__ __forceinline__ int sum_pm1(const uint32_t (&a)[4]) {
  return 2 * (__popc(a[0]) + __popc(a[1]) + __popc(a[2]) + __popc(a[3])) - kQuantGroup;
}

// Exact sums sum(b_i w) of the first P planes, i = 0..P-1.
template <int P>
__device__ __forceinline__ void signed_sums(const double (&w)[kSlots], const unsigned (&code)[kSlots],
                                            double (&S)[P]) {
  double t[P];
#pragma unroll
  for (int i = 0; i < P; ++i) {
    t[i] = 0.0;
#pragma unroll
    for (int s = 0; s < kSlots; ++s) t[i] += signed_val((code[s] >> i) & 1u, w[s]);
  }
#pragma unroll
  for (int i = 0; i + 1 < P; i += 2) group_sum2_exact(t[i], t[i + 1], S[i], S[i + 1]);
  if constexpr (P % 2 == 1) S[P - 1] = group_sum(t[P - 1]);
}

// Joint least squares for (z, alpha_1..alpha_P): columns [ones, b_1..b_P],
// right-hand sides sum(w) and sum(b_i w).
template <int P>
__device__ __forceinline__ void lsq_with_offset(const double (&w)[kSlots], double sumw,
                                                const unsigned (&code)[kSlots], double (&alpha)[P],
                                                double& z) {
  uint32_t pw[P][4];
  plane_words<P>(code, pw);
  int G[P + 1][P + 1];
  double r[P + 1], x[P + 1], S[P];
  signed_sums<P>(w, code, S);
  G[0][0] = kQuantGroup;
  r[0] = sumw;
#pragma unroll
  for (int i = 0; i < P; ++i) {
    G[0][i + 1] = G[i + 1][0] = sum_pm1(pw[i]);
#pragma unroll
    for (int j = 0; j <= i; ++j) G[i + 1][j + 1] = G[j + 1][i + 1] = dot_pm1(pw[i], pw[j]);
    r[i + 1] = S[i];
  }
  solve_exact<P + 1>(G, r, x);
  z = x[0];
#pragma unroll
  for (int i = 0; i < P; ++i) alpha[i] = x[i + 1];
}

// Least squares for alpha_1..alpha_P with z fixed: columns [b_1..b_P],
// right-hand sides sum(b_i (w - z)) = sum(b_i w) - z sum(b_i).
template <int P>
__device__ __forceinline__ void lsq_fixed_offset(const double (&w)[kSlots], double z,
                                                 const unsigned (&code)[kSlots], double (&alpha)[P]) {
  uint32_t pw[P][4];
  plane_words<P>(code, pw);
  int G[P][P];
  double r[P], S[P];
  signed_sums<P>(w, code, S);
#pragma unroll
  for (int i = 0; i < P; ++i) {
#pragma unroll
    for (int j = 0; j <= i; ++j) G[i][j] = G[j][i] = dot_pm1(pw[i], pw[j]);
    r[i] = __dsub_rn(S[i], __dmul_rn(z, (double)sum_pm1(pw[i])));
  }
  solve_exact<P>(G, r, alpha);
}

// z + (((alpha_1 b_1) + alpha_2 b_2) + ...) for code c.
template <int P>
__device__ __forceinline__ double code_value(const double (&alpha)[P], double z, unsigned c) {
  double acc = signed_val(c & 1u, alpha[0]);
#pragma unroll
  for (int i = 1; i < P; ++i) acc += signed_val((c >> i) & 1u, alpha[i]);
  return z + acc;
}

template <int P>
__device__ __forceinline__ void nearest_codes(const double (&w)[kSlots], const double (&alpha)[P],
                                              double z, unsigned (&code)[kSlots]) {
  constexpr int C = 1 << P;
  double v[C];
#pragma unroll
  for (int c = 0; c < C; ++c) v[c] = code_value<P>(alpha, z, (unsigned)c);
#pragma unroll
  for (int s = 0; s < kSlots; ++s) {
    unsigned best = 0;
    double be = fabs(w[s] - v[0]);
#pragma unroll
    for (int c = 1; c < C; ++c) {
      const double e = fabs(w[s] - v[c]);
      if (e < be) {
        be = e;
        best = (unsigned)c;
      }
    }
    code[s] = best;
  }
}

template <int P>
__device__ __forceinline__ double group_sse(const double (&w)[kSlots], const double (&alpha)[P],
                                            double z, const unsigned (&code)[kSlots]) {
  double t = 0.0;
#pragma unroll
  for (int s = 0; s < kSlots; ++s) {
    const double e = w[s] - code_value<P>(alpha, z, code[s]);
    t += e * e;
  }
  return group_sum(t);
}

// alpha^(P) of the group rounded to fp16 (nearest even), and its error;
// j = the lane within the group, valid = the lanes hold a real group.
template <int P>
__device__ __forceinline__ void store_scales(const QuantParams& q, long long gid, int j,
                                             bool valid, const double (&alpha)[P], double sse,
                                             int p_L) {
  if (!valid) return;
  __half* a = q.alpha[P - 1] + gid * P;
#pragma unroll
  for (int i = 0; i < P; ++i)
    if (j == i) a[i] = __double2half(alpha[i]);
  if (q.sse && j == 0) q.sse[(long long)(P - p_L) * q.groups + gid] = sse;
}

// Base precision PL: greedy start, refinement rounds, final refit.
template <int PL>
__device__ __forceinline__ void base_precision(const QuantParams& q, const double (&w)[kSlots],
                                               double sumw, unsigned (&code)[kSlots],
                                               double (&alpha)[PL], double& z) {
  z = sumw / kQuantGroup;  // exact: the sum is exact, 128 a power of two
  double r[kSlots];
#pragma unroll
  for (int s = 0; s < kSlots; ++s) {
    r[s] = w[s] - z;
    code[s] = 0;
  }
  uint32_t pw[PL][4];
#pragma unroll
  for (int i = 0; i < PL; ++i) {
#pragma unroll
    for (int s = 0; s < kSlots; ++s) code[s] |= (r[s] >= 0.0 ? 1u : 0u) << i;  // b_i = sign(r)
    plane_word(code, i, pw[i]);
    // <b_i, r> = sum(b_i w) - z sum(b_i) - sum_j alpha_j <b_i, b_j>, left to right
    double t = 0.0;
#pragma unroll
    for (int s = 0; s < kSlots; ++s) t += signed_val((code[s] >> i) & 1u, w[s]);
    t = group_sum(t);
    t = __dsub_rn(t, __dmul_rn(z, (double)sum_pm1(pw[i])));
#pragma unroll
    for (int j = 0; j < i; ++j) t = __dsub_rn(t, __dmul_rn(alpha[j], (double)dot_pm1(pw[i], pw[j])));
    const double a = t / kQuantGroup;
#pragma unroll
    for (int s = 0; s < kSlots; ++s) r[s] = ((code[s] >> i) & 1u) ? r[s] - a : r[s] + a;
    alpha[i] = a;
  }
  for (int it = 0; it < q.rounds; ++it) {
    lsq_with_offset<PL>(w, sumw, code, alpha, z);
    nearest_codes<PL>(w, alpha, z, code);
  }
  lsq_with_offset<PL>(w, sumw, code, alpha, z);
}

// Expansion p -> p + 1: B_{p+1} = sign(R_p), then every scale refit with z
// kept (shared offsets) or refit with it (q.zp: offsets per precision).
template <int P, int PH, bool ZP>
__device__ __forceinline__ void expand(const QuantParams& q, long long gid, int j, bool valid,
                                       int p_L,
                                       const double (&w)[kSlots], double sumw, double z,
                                       unsigned (&code)[kSlots], const double (&alpha)[P]) {
  if constexpr (P < PH) {
#pragma unroll
    for (int s = 0; s < kSlots; ++s) {
      const double res = w[s] - code_value<P>(alpha, z, code[s]);
      code[s] |= (res >= 0.0 ? 1u : 0u) << P;
    }
    double next[P + 1];
    double zn = z;
    if constexpr (ZP) {
      lsq_with_offset<P + 1>(w, sumw, code, next, zn);
      if (valid && j == 0) q.zq[P][gid] = __double2half(zn);
    } else {
      lsq_fixed_offset<P + 1>(w, z, code, next);
    }
    const double e = q.sse ? group_sse<P + 1>(w, next, zn, code) : 0.0;
    store_scales<P + 1>(q, gid, j, valid, next, e, p_L);
    expand<P + 1, PH, ZP>(q, gid, j, valid, p_L, w, sumw, zn, code, next);
  }
}

template <int PL, int PH, bool ZP>
__global__ void __launch_bounds__(32 * kQuantWarps, kQuantMinCtas) quantize_kernel(QuantParams q) {
  const int j = threadIdx.x & (kGroupLanes - 1);
  const long long gid0 = ((long long)blockIdx.x * kQuantWarps + (threadIdx.x >> 5)) * 4;
  if (gid0 >= q.groups) return;  // uniform per warp
  const long long gid = gid0 + ((threadIdx.x >> 3) & 3);
  // the last warp may hold fewer than four groups: a lane without a group
  // computes on the warp's first group (every lane takes part in the
  // ballots and shuffles) and stores nothing
  const bool valid = gid < q.groups;
  const long long gl = valid ? gid : gid0;
  const long long n = gl / q.G;
  const int g = (int)(gl - n * q.G);
  const __half* src = q.w + n * q.K + (long long)g * kQuantGroup;
  double w[kSlots];
#pragma unroll
  for (int s = 0; s < kSlots; ++s) w[s] = (double)__half2float(src[j + kGroupLanes * s]);
  double tw = 0.0;
#pragma unroll
  for (int s = 0; s < kSlots; ++s) tw += w[s];
  const double sumw = group_sum(tw);  // exact in any order

  unsigned code[kSlots];
  double alpha[PL], z;
  base_precision<PL>(q, w, sumw, code, alpha, z);
  const double e = q.sse ? group_sse<PL>(w, alpha, z, code) : 0.0;
  store_scales<PL>(q, gid, j, valid, alpha, e, PL);
  if (valid && j == 0) (ZP ? q.zq[PL - 1] : q.z)[gid] = __double2half(z);
  expand<PL, PH, ZP>(q, gid, j, valid, PL, w, sumw, z, code, alpha);

  // planes: lane (4 i + t) mod 8 of the group writes word t of plane i
  uint32_t pw[PH][4];
  plane_words<PH>(code, pw);
  const int KW = q.K / 32;
#pragma unroll
  for (int i = 0; i < PH; ++i)
#pragma unroll
    for (int t = 0; t < 4; ++t)
      if (valid && j == ((4 * i + t) & 7)) q.planes[((long long)i * q.N + n) * KW + 4 * g + t] = pw[i][t];
}

using QuantKernel = void (*)(QuantParams);

QuantKernel quantize_kernel_for(int p_L, int p_H, bool zp) {
#define BCQ_Q(a, b) \
  if (p_L == a && p_H == b) return zp ? quantize_kernel<a, b, true> : quantize_kernel<a, b, false>;
  BCQ_Q(1, 1) BCQ_Q(1, 2) BCQ_Q(1, 3) BCQ_Q(1, 4)
  BCQ_Q(2, 2) BCQ_Q(2, 3) BCQ_Q(2, 4)
  BCQ_Q(3, 3) BCQ_Q(3, 4)
  BCQ_Q(4, 4)
#undef BCQ_Q
  return nullptr;
}

bool aligned_to(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace
}  // namespace bcq

namespace bcq {
namespace {

bcq_status quantize_common(const uint16_t* w, int N, int K, int p_L, int p_H, int rounds,
                           uint32_t* planes, uint16_t* const alpha[4], uint16_t* z,
                           uint16_t* const zq[4], double* sse, void* stream) {
  if (!alpha) return BCQ_ERR_NULL;
  if (p_H < 1 || p_H > BCQ_MAX_PLANES || p_L < 1 || p_L > p_H) return BCQ_ERR_PRECISION;
  if (N < 0 || K < 0 || K % BCQ_GROUP != 0 || rounds < 0 || rounds > 1000) return BCQ_ERR_SHAPE;
  if ((long long)N * (K / BCQ_GROUP) > (1ll << 33)) return BCQ_ERR_SHAPE;
  if (N == 0 || K == 0) return BCQ_OK;
  if (!w || !planes || (!z && !zq)) return BCQ_ERR_NULL;
  for (int p = p_L; p <= p_H; ++p) {
    if (!alpha[p - 1]) return BCQ_ERR_PRECISION;
    if (zq && !zq[p - 1]) return BCQ_ERR_NULL;
  }
  if (!aligned_to(w, 2) || !aligned_to(planes, 4) || (z && !aligned_to(z, 2)) ||
      (sse && !aligned_to(sse, 8)))
    return BCQ_ERR_ALIGN;
  for (int p = p_L; p <= p_H; ++p)
    if (!aligned_to(alpha[p - 1], 2) || (zq && !aligned_to(zq[p - 1], 2))) return BCQ_ERR_ALIGN;
  QuantParams q{};
  q.w = reinterpret_cast<const __half*>(w);
  q.planes = planes;
  for (int p = 1; p <= 4; ++p) {
    const bool used = p >= p_L && p <= p_H;
    q.alpha[p - 1] = used ? reinterpret_cast<__half*>(alpha[p - 1]) : nullptr;
    q.zq[p - 1] = used && zq ? reinterpret_cast<__half*>(zq[p - 1]) : nullptr;
  }
  q.z = reinterpret_cast<__half*>(z);
  q.sse = sse;
  q.N = N;
  q.K = K;
  q.G = K / BCQ_GROUP;
  q.groups = (long long)N * q.G;
  q.rounds = rounds;
  const QuantKernel fn = quantize_kernel_for(p_L, p_H, zq != nullptr);
  if (!fn) return BCQ_ERR_UNSUPPORTED;
  const long long blocks = (q.groups + 4 * kQuantWarps - 1) / (4 * kQuantWarps);
  fn<<<(unsigned)blocks, 32 * kQuantWarps, 0, (cudaStream_t)stream>>>(q);
  return cudaGetLastError() == cudaSuccess ? BCQ_OK : BCQ_ERR_CUDA;
}

}  // namespace
}  // namespace bcq

extern "C" bcq_status bcq_quantize(const uint16_t* w, int N, int K, int p_L, int p_H,
                                   int rounds, uint32_t* planes, uint16_t* const alpha[4],
                                   uint16_t* z, double* sse, void* stream) {
  if (!z && N > 0 && K > 0) return BCQ_ERR_NULL;
  return bcq::quantize_common(w, N, K, p_L, p_H, rounds, planes, alpha, z, nullptr, sse, stream);
}

extern "C" bcq_status bcq_quantize_zp(const uint16_t* w, int N, int K, int p_L, int p_H,
                                      int rounds, uint32_t* planes, uint16_t* const alpha[4],
                                      uint16_t* const z[4], double* sse, void* stream) {
  if (!z && N > 0 && K > 0) return BCQ_ERR_NULL;
  return bcq::quantize_common(w, N, K, p_L, p_H, rounds, planes, alpha, nullptr, z, sse, stream);
}
