// kvq_fft.cuh -- the SRFT's complex FFT building blocks, shared by the codec
// (kvq_srft.cuh) and the decode attention (kvq_attn.cu): products by
// twiddles with the exact rounding the oracle states, Stockham stages of
// radix 2 and 3 on register arrays and their transposes, the Hermitian
// unpacking of one lane's vector and its adjoint, and the host's table of
// correctly rounded roots of unity.  Included inside a translation unit's
// anonymous namespace, after kvq_arith.cuh.
#pragma once

// ---- compile-time loops and twiddle products -----------------------------

template <int I, int E, typename Fn>
__device__ __forceinline__ void sfor(Fn&& f) {
  if constexpr (I < E) {
    f(std::integral_constant<int, I>{});
    sfor<I + 1, E>(f);
  }
}

// d * omega_M^K, or d * conj(omega_M^K) (CONJ), K known at compile time; w is
// the table of omega_M.  A product by 1, -1, i or -i is exact (the operand,
// negated or with its parts swapped); any other is one rounded product and
// one fused multiply-add per part: re = fma(d.x, w.x, -rn(d.y w.y)),
// im = fma(d.y, w.x, rn(d.x w.y)).
template <int K, int M, bool CONJ>
__device__ __forceinline__ float2 twmul(float2 d, const float2* w) {
  constexpr int k = K % M;
  if constexpr ((4 * k) % M == 0) {                       // 1, -i, -1, i: exact
    constexpr int e = CONJ ? (4 - (4 * k) / M) % 4 : (4 * k) / M;   // w = (-i)^e
    if constexpr (e == 0) return d;
    else if constexpr (e == 1) return make_float2(d.y, -d.x);
    else if constexpr (e == 2) return make_float2(-d.x, -d.y);
    else return make_float2(-d.y, d.x);
  } else {
    const float2 t = w[k];
    const float ty = CONJ ? -t.y : t.y;
    const float b = __fmul_rn(d.y, ty), c = __fmul_rn(d.x, ty);
    return make_float2(__fmaf_rn(d.x, t.x, -b), __fmaf_rn(d.y, t.x, c));
  }
}

// omega_M^K (d / i), the forward unpacking's odd part, d / i = (d.y, -d.x):
// re = fma(d.y, wx, rn(d.x wy)), im = fma(-d.x, wx, rn(d.y wy)), the same
// roundings as the product of (d / i) and w.
template <int K, int M>
__device__ __forceinline__ float2 twmul_odiv(float2 d, const float2* w) {
  constexpr int k = K % M;
  if constexpr ((4 * k) % M == 0) {
    return twmul<K, M, false>(make_float2(d.y, -d.x), w);
  } else {
    const float2 t = w[k];
    const float p = __fmul_rn(d.x, t.y), q = __fmul_rn(d.y, t.y);
    return make_float2(__fmaf_rn(d.y, t.x, p), __fmaf_rn(-d.x, t.x, q));
  }
}
// The same with a twiddle known only at run time (never 1, -1, i or -i).
__device__ __forceinline__ float2 twmul_odiv_rt(float2 d, float2 t) {
  const float p = __fmul_rn(d.x, t.y), q = __fmul_rn(d.y, t.y);
  return make_float2(__fmaf_rn(d.y, t.x, p), __fmaf_rn(-d.x, t.x, q));
}
__device__ __forceinline__ float2 twmul_conj_rt(float2 d, float2 t) {
  const float ty = -t.y;
  const float b = __fmul_rn(d.y, ty), c = __fmul_rn(d.x, ty);
  return make_float2(__fmaf_rn(d.x, t.x, -b), __fmaf_rn(d.y, t.x, c));
}

// ---- Stockham stages on an L-point register array -------------------------
// The twiddles of the L-point transform are omega_L^j = omega_M^(j M / L),
// read from the table of omega_M.

// Forward radix 2, sub-transforms of length n, stride s = L / n:
// y[q + 2sp] = a + b, y[q + s(2p+1)] = (a - b) omega_n^p,
// a = x[q + sp], b = x[q + s(p + n/2)].
template <int L, int n, int M>
__device__ __forceinline__ void dif2(float2 (&x)[L], const float2* w) {
  constexpr int s = L / n, m = n / 2;
  float2 y[L];
  sfor<0, m>([&](auto P) {
    constexpr int p = decltype(P)::value;
    sfor<0, s>([&](auto Qi) {
      constexpr int q = decltype(Qi)::value;
      const float2 a = x[q + s * p], b = x[q + s * (p + m)];
      y[q + s * 2 * p] = __fadd2_rn(a, b);
      y[q + s * (2 * p + 1)] = twmul<p * s * (M / L), M, false>(fsub2(a, b), w);
    });
  });
#pragma unroll
  for (int i = 0; i < L; ++i) x[i] = y[i];
}

// Forward radix 3 (the last stage, n = 3, stride s = L / 3):
// y[q + s t] = (a0 + omega_3^t a1) + omega_3^2t a2.
template <int L, int M>
__device__ __forceinline__ void dif3(float2 (&x)[L], const float2* w) {
  constexpr int s = L / 3, K3 = M / 3;
  float2 y[L];
  sfor<0, s>([&](auto Qi) {
    constexpr int q = decltype(Qi)::value;
    const float2 a0 = x[q], a1 = x[q + s], a2 = x[q + 2 * s];
    y[q] = __fadd2_rn(__fadd2_rn(a0, a1), a2);
    y[q + s] = __fadd2_rn(__fadd2_rn(a0, twmul<K3, M, false>(a1, w)), twmul<2 * K3, M, false>(a2, w));
    y[q + 2 * s] = __fadd2_rn(__fadd2_rn(a0, twmul<2 * K3, M, false>(a1, w)), twmul<4 * K3, M, false>(a2, w));
  });
#pragma unroll
  for (int i = 0; i < L; ++i) x[i] = y[i];
}

// The transposes (inverse): radix 2, c = y[q + s(2p+1)] conj(omega_n^p),
// x[q + sp] = y[q + 2sp] + c, x[q + s(p + n/2)] = y[q + 2sp] - c.
template <int L, int n, int M>
__device__ __forceinline__ void dit2(float2 (&x)[L], const float2* w) {
  constexpr int s = L / n, m = n / 2;
  float2 y[L];
  sfor<0, m>([&](auto P) {
    constexpr int p = decltype(P)::value;
    sfor<0, s>([&](auto Qi) {
      constexpr int q = decltype(Qi)::value;
      const float2 a = x[q + s * 2 * p];
      const float2 c = twmul<p * s * (M / L), M, true>(x[q + s * (2 * p + 1)], w);
      y[q + s * p] = __fadd2_rn(a, c);
      y[q + s * (p + m)] = fsub2(a, c);
    });
  });
#pragma unroll
  for (int i = 0; i < L; ++i) x[i] = y[i];
}

// Radix 3: x[q + s j] = (c0 + conj(omega_3^j) c1) + conj(omega_3^2j) c2.
template <int L, int M>
__device__ __forceinline__ void dit3(float2 (&x)[L], const float2* w) {
  constexpr int s = L / 3, K3 = M / 3;
  float2 y[L];
  sfor<0, s>([&](auto Qi) {
    constexpr int q = decltype(Qi)::value;
    const float2 c0 = x[q], c1 = x[q + s], c2 = x[q + 2 * s];
    y[q] = __fadd2_rn(__fadd2_rn(c0, c1), c2);
    y[q + s] = __fadd2_rn(__fadd2_rn(c0, twmul<K3, M, true>(c1, w)), twmul<2 * K3, M, true>(c2, w));
    y[q + 2 * s] = __fadd2_rn(__fadd2_rn(c0, twmul<2 * K3, M, true>(c1, w)), twmul<4 * K3, M, true>(c2, w));
  });
#pragma unroll
  for (int i = 0; i < L; ++i) x[i] = y[i];
}

template <int L, int n, int M>
__device__ __forceinline__ void fft_fwd_from(float2 (&x)[L], const float2* w) {
  if constexpr (n % 2 == 0) {
    dif2<L, n, M>(x, w);
    fft_fwd_from<L, n / 2, M>(x, w);
  } else if constexpr (n == 3) {
    dif3<L, M>(x, w);
  }
}
template <int L, int n, int M>
__device__ __forceinline__ void fft_inv_from(float2 (&x)[L], const float2* w) {
  if constexpr (n % 2 == 0) {
    fft_inv_from<L, n / 2, M>(x, w);
    dit2<L, n, M>(x, w);
  } else if constexpr (n == 3) {
    dit3<L, M>(x, w);
  }
}

// ---- the Hermitian unpacking, one lane per vector (D <= 128) ---------------
// In place on z[N]: z[0] -> (y0, y1), z[k] -> (y_2k, y_2k+1).  fac(n) gives
// the factors of positions 2n, 2n+1 (the odd one negated above N/2).
template <int D, typename Fac>
__device__ __forceinline__ void unpack_fwd1(float2 (&z)[D / 2], const float2* wd, Fac fac) {
  constexpr int N = D / 2;
  const float2 z0 = z[0];
  z[0] = __fmul2_rn(make_float2(__fadd_rn(z0.x, z0.y), __fsub_rn(z0.x, z0.y)), fac(0));
  sfor<1, N / 2 + 1>([&](auto Kc) {
    constexpr int k = decltype(Kc)::value;
    const float2 A = z[k], Bz = z[N - k];
    const float2 E = __ffma2_rn(Bz, make_float2(1.0f, -1.0f), A);     // A + conj Bz
    const float2 Dd = __ffma2_rn(Bz, make_float2(-1.0f, 1.0f), A);    // A - conj Bz
    const float2 T = twmul_odiv<k, D>(Dd, wd);
    z[k] = __fmul2_rn(__fadd2_rn(E, T), fac(k));
    if constexpr (2 * k < N) z[N - k] = __fmul2_rn(fsub2(E, T), fac(N - k));
  });
}

// The adjoint, in place: z[n] holds (u_2n, u_2n+1); fac(n) the factors of
// positions 2n, 2n+1.  Afterwards z is the half-length spectrum Z.
template <int D, typename Fac>
__device__ __forceinline__ void unpack_inv1(float2 (&z)[D / 2], const float2* wd, Fac fac) {
  constexpr int N = D / 2;
  const float2 u0 = __fmul2_rn(z[0], fac(0));                          // (U_0, U_N)
  z[0] = make_float2(__fadd_rn(u0.x, u0.y), __fsub_rn(u0.x, u0.y));
  sfor<1, N / 2 + 1>([&](auto Kc) {
    constexpr int k = decltype(Kc)::value;
    const float2 A = __fmul2_rn(z[k], fac(k));
    float2 Bu = A;
    if constexpr (2 * k < N) Bu = __fmul2_rn(z[N - k], fac(N - k));
    const float2 E = __ffma2_rn(Bu, make_float2(1.0f, -1.0f), A);     // A + conj Bu
    const float2 Dd = __ffma2_rn(Bu, make_float2(-1.0f, 1.0f), A);    // A - conj Bu
    const float2 T = twmul<k, D, true>(Dd, wd);
    z[k] = make_float2(__fsub_rn(E.x, T.y), __fadd_rn(E.y, T.x));     // E + iT
    if constexpr (2 * k < N)
      z[N - k] = make_float2(__fadd_rn(E.x, T.y), -__fsub_rn(E.y, T.x));   // conj(E - iT)
  });
}


// ---- the host's twiddle table -------------------------------------------------

// omega_M^k = (cos, -sin)(2 pi k / M), each part the fp32 value nearest the
// exact one: the angle is reduced by exact symmetries (quadrant, then the
// complement within it) to at most pi/4, whose cosine and sine are evaluated
// in long double and rounded once; zero parts are +0.
float2 root_f32(int k, int M) {
  const long j = (static_cast<long>(k) % M + M) % M;
  const long q = 4 * j / M, r0 = 4 * j - q * M;
  const bool comp = 2 * r0 > M;
  const long r = comp ? M - r0 : r0;
  const long double ang = 1.57079632679489661923132169163975144L * static_cast<long double>(r) /
                          static_cast<long double>(M);
  float c = static_cast<float>(cosl(ang)), s = static_cast<float>(sinl(ang));
  if (comp) { const float t = c; c = s; s = t; }
  float cr, sn;
  switch (q) {
    case 0: cr = c; sn = s; break;
    case 1: cr = -s; sn = c; break;
    case 2: cr = -c; sn = -s; break;
    default: cr = s; sn = -c; break;
  }
  return make_float2(cr + 0.0f, -sn + 0.0f);     // -0 -> +0
}

