// cells.cuh -- the three diagonal cells, one channel at a time, in float32.
//
// Each cell provides
//   warm(p, w, f)                  f = f(0, x): the Newton warm start
//                                  (pararnn-torch PyPI page, Method section,
//                                  "h^(0) = f(0, x)")
//   elem(p, w, sp, f, A, beta)     f = f(sp, x), A = df/dsp (S x S, row-major),
//                                  beta = f - A sp: the scan element of the
//                                  direct-form Newton update
//                                  h_t = A_t h_{t-1} + beta_t
//   bwd(p, w, sp, A, sens)         A and the sensitivities the adjoint needs
//   grads(sens, lam, dp, da)       dL/dp_g and dL/da_g of one row given
//                                  lambda_t (the adjoint state)
// Cell equations: diagonal GRU (gates z, r, c) and diagonal LSTM (gates i, f,
// o, c; forget bias +1; state (c, h)) as listed for ParaGRU / ParaLSTM on the
// pararnn-torch page; the linear cell h' = a h + b is the affine recurrence
// the News section calls an exact parallel scan.
#pragma once

#include "common.cuh"

namespace pararnn {

struct CellLinear {
    static constexpr int G = 2, S = 1, NSENS = 1;
    static constexpr bool kNonlinear = false;  // one scan is exact
    struct W2 {};  // no packed form: the linear cell's arithmetic is one FMA per row

    static __device__ __forceinline__ void warm(const float (&p)[G], const float (&)[G], float (&f)[S]) {
        f[0] = p[1];
    }
    static __device__ __forceinline__ void elem(const float (&p)[G], const float (&)[G], const float (&sp)[S],
                                                float (&f)[S], float (&A)[S * S], float (&beta)[S]) {
        A[0] = p[0];
        beta[0] = p[1];
        f[0] = __fmaf_rn(p[0], sp[0], p[1]);
    }
    static __device__ __forceinline__ void bwd(const float (&p)[G], const float (&)[G], const float (&sp)[S],
                                               float (&A)[S * S], float (&sens)[NSENS]) {
        A[0] = p[0];
        sens[0] = sp[0];
    }
    static __device__ __forceinline__ void grads(const float (&sens)[NSENS], const float (&lam)[S], float (&dp)[G],
                                                 float (&da)[G]) {
        dp[0] = lam[0] * sens[0];
        dp[1] = lam[0];
        da[0] = 0.0f;
        da[1] = 0.0f;
    }
};

struct CellGRU {
    static constexpr int G = 3, S = 1, NSENS = 5;
    static constexpr bool kNonlinear = true;

    static __device__ __forceinline__ void warm(const float (&p)[G], const float (&)[G], float (&f)[S]) {
        // h = 0: z = sig(p_z), c = tanh(p_c), f = z c; z and c share a reciprocal
        float z, ic;
        inv_pair(sig_den(p[0]), tanh_den(p[2]), z, ic);
        f[0] = z * tanh_from_inv(p[2], ic);
    }
    // z, r, c and the chain-rule factors G_z = df/dp_z, G_r = df/dp_r, G_c = df/dp_c
    static __device__ __forceinline__ void gates(const float (&p)[G], const float (&w)[G], float h, float& z,
                                                 float& r, float& c, float& Gz, float& Gr, float& Gc) {
        z = sigmoid_f(__fmaf_rn(w[0], h, p[0]));
        r = sigmoid_f(__fmaf_rn(w[1], h, p[1]));
        c = tanh_f(__fmaf_rn(w[2] * r, h, p[2]));
        Gz = (c - h) * (z - z * z);
        Gc = z * __fmaf_rn(-c, c, 1.0f);
        Gr = Gc * w[2] * h * (r - r * r);
    }
    static __device__ __forceinline__ void elem(const float (&p)[G], const float (&w)[G], const float (&sp)[S],
                                                float (&f)[S], float (&A)[S * S], float (&beta)[S]) {
        const float h = sp[0];
        // the update and reset gates share a reciprocal; the candidate
        // depends on r and takes its own
        float z, r;
        inv_pair(sig_den(__fmaf_rn(w[0], h, p[0])), sig_den(__fmaf_rn(w[1], h, p[1])), z, r);
        const float wr = w[2] * r;
        const float c = tanh_f(__fmaf_rn(wr, h, p[2]));
        const float ch = c - h;
        f[0] = __fmaf_rn(z, ch, h);  // (1 - z) h + z c
        // df/dh = (1 - z) + a_z G_z + a_r G_r + a_c r G_c with G_z = (c - h) z (1 - z),
        // G_c = z (1 - c^2), G_r = G_c a_c h r (1 - r); the last two share G_c a_c:
        //   a_r G_r + a_c r G_c = G_c a_c (a_r h r (1 - r) + r)
        const float gcw = z * __fmaf_rn(-c, c, 1.0f) * w[2];
        const float tr = __fmaf_rn(w[1] * h, __fmaf_rn(-r, r, r), r);
        float a = __fmaf_rn(w[0], ch * __fmaf_rn(-z, z, z), 1.0f - z);
        a = __fmaf_rn(gcw, tr, a);
        A[0] = a;
        beta[0] = __fmaf_rn(-a, h, f[0]);
    }
    // ---- two channels per instruction (packed f32x2) ----
    // the recurrent weights of a channel pair, with the negated copy the
    // sign-free algebra below needs
    struct W2 {
        f2 w0, w1, w2, nw2;
    };
    static __device__ __forceinline__ W2 weights2(const float (&wa)[G], const float (&wb)[G]) {
        return W2{f2{wa[0], wb[0]}, f2{wa[1], wb[1]}, f2{wa[2], wb[2]}, f2{-wa[2], -wb[2]}};
    }
    // warm() on a pair of channels
    static __device__ __forceinline__ void warm2(const f2 (&p)[G], f2 (&f)[S]) {
        f2 z, ic;
        inv_pair2(sig_den2(p[0]), tanh_den2(p[2]), z, ic);
        f[0] = mul2(z, tanh2_from_inv(p[2], ic));
    }
    // elem() on a pair of channels.  No packed negation exists, so the gates
    // are formed negated, nz = -z and nr = -r (from negated denominators), and every sign
    // is carried by the algebra:
    //   f      = z (c - h) + h            = nz (h - c) + h
    //   a_c r  = (-a_c) nr
    //   G_z a_z= a_z (c - h)(z - z^2)     = a_z (h - c)(nz^2 + nz)
    //   1 - z  = 1 + nz
    //   the shared reset/candidate term  G_c a_c (a_r h r (1 - r) + r)
    //          = (nz (c^2 - 1) (-a_c)) * (a_r h (nr^2 + nr) + nr)
    // Each product or sum is the same floating-point operation as in elem()
    // up to the sign of its operands, so each result is elem()'s, negated
    // where the algebra says so.
    static __device__ __forceinline__ void elem2(const f2 (&p)[G], const W2& w, const f2 (&sp)[S], f2 (&f)[S],
                                                 f2 (&A)[S * S], f2 (&beta)[S]) {
        elem2(p, w, sp[0], f[0], A[0], beta[0]);
    }
    static __device__ __forceinline__ void elem2(const f2 (&p)[G], const W2& w, f2 h, f2& f, f2& A, f2& beta) {
        // -z and -r from one reciprocal of (-1 - e_z)(-1 - e_r), which is
        // the product elem() inverts, exactly
        f2 nz, nr;
        inv_pair2(neg_sig_den2(fma2(w.w0, h, p[0])), neg_sig_den2(fma2(w.w1, h, p[1])), nz, nr);
        const f2 wr = mul2(w.nw2, nr);
        const f2 c = tanh2(fma2(wr, h, p[2]));
        const f2 hc = sub2(h, c);
        f = fma2(nz, hc, h);
        const f2 ngcw = mul2(mul2(nz, fma2(c, c, splat2(-1.0f))), w.nw2);
        const f2 ntr = fma2(mul2(w.w1, h), fma2(nr, nr, nr), nr);
        f2 a = fma2(w.w0, mul2(hc, fma2(nz, nz, nz)), add2(splat2(1.0f), nz));
        a = fma2(ngcw, ntr, a);
        A = a;
        beta = fma2(a, mul2(h, splat2(-1.0f)), f);
    }
    // bwd() on a pair of channels, with the negated gates of elem2():
    //   G_z = (c - h)(z - z^2)      = (h - c)(nz^2 + nz)
    //   G_c = z (1 - c^2)           = nz (c^2 - 1)
    //   G_r = G_c a_c h (r - r^2)   = ((G_c (-a_c)) h)(nr^2 + nr)
    //   r h = -(nr h)
    static __device__ __forceinline__ void bwd2(const f2 (&p)[G], const W2& w, const f2 (&sp)[S], f2 (&A)[S * S],
                                                f2 (&sens)[NSENS]) {
        const f2 h = sp[0], mone = splat2(-1.0f);
        const f2 nz = neg_sigmoid2(fma2(w.w0, h, p[0]));
        const f2 nr = neg_sigmoid2(fma2(w.w1, h, p[1]));
        const f2 wr = mul2(w.nw2, nr);
        const f2 c = tanh2(fma2(wr, h, p[2]));
        const f2 Gz = mul2(sub2(h, c), fma2(nz, nz, nz));
        const f2 Gc = mul2(nz, fma2(c, c, mone));
        const f2 Gr = mul2(mul2(mul2(Gc, w.nw2), h), fma2(nr, nr, nr));
        f2 a = add2(splat2(1.0f), nz);
        a = fma2(w.w0, Gz, a);
        a = fma2(w.w1, Gr, a);
        a = fma2(wr, Gc, a);
        A[0] = a;
        sens[0] = Gz;
        sens[1] = Gr;
        sens[2] = Gc;
        sens[3] = mul2(mul2(nr, h), mone);
        sens[4] = h;
    }
    static __device__ __forceinline__ void grads2(const f2 (&sens)[NSENS], const f2 (&lam)[S], f2 (&dp)[G],
                                                  f2 (&da)[G]) {
        dp[0] = mul2(lam[0], sens[0]);
        dp[1] = mul2(lam[0], sens[1]);
        dp[2] = mul2(lam[0], sens[2]);
        da[0] = mul2(dp[0], sens[4]);
        da[1] = mul2(dp[1], sens[4]);
        da[2] = mul2(dp[2], sens[3]);
    }
    static __device__ __forceinline__ void bwd(const float (&p)[G], const float (&w)[G], const float (&sp)[S],
                                               float (&A)[S * S], float (&sens)[NSENS]) {
        const float h = sp[0];
        float z, r, c, Gz, Gr, Gc;
        gates(p, w, h, z, r, c, Gz, Gr, Gc);
        float a = 1.0f - z;
        a = __fmaf_rn(w[0], Gz, a);
        a = __fmaf_rn(w[1], Gr, a);
        a = __fmaf_rn(w[2] * r, Gc, a);
        A[0] = a;
        sens[0] = Gz;
        sens[1] = Gr;
        sens[2] = Gc;
        sens[3] = r * h;
        sens[4] = h;
    }
    static __device__ __forceinline__ void grads(const float (&sens)[NSENS], const float (&lam)[S], float (&dp)[G],
                                                 float (&da)[G]) {
        dp[0] = lam[0] * sens[0];
        dp[1] = lam[0] * sens[1];
        dp[2] = lam[0] * sens[2];
        da[0] = dp[0] * sens[4];
        da[1] = dp[1] * sens[4];
        da[2] = dp[2] * sens[3];
    }
};

struct CellLSTM {
    static constexpr int G = 4, S = 2, NSENS = 6;
    static constexpr bool kNonlinear = true;

    static __device__ __forceinline__ void warm(const float (&p)[G], const float (&)[G], float (&f)[S]) {
        // (c, h) = 0: c' = i g, h' = o tanh(c')
        const float i = sigmoid_f(p[0]);
        const float o = sigmoid_f(p[2]);
        const float g = tanh_f(p[3]);
        const float cn = i * g;
        f[0] = cn;
        f[1] = o * tanh_f(cn);
    }
    struct Terms {
        float i, fg, o, g, ig, cn, tn, dcn_dh;
    };
    static __device__ __forceinline__ Terms terms(const float (&p)[G], const float (&w)[G], float c, float h) {
        Terms q;
        q.i = sigmoid_f(__fmaf_rn(w[0], h, p[0]));
        q.fg = sigmoid_f(__fmaf_rn(w[1], h, p[1]) + 1.0f);
        q.o = sigmoid_f(__fmaf_rn(w[2], h, p[2]));
        q.g = tanh_f(__fmaf_rn(w[3], h, p[3]));
        q.ig = q.i * q.g;
        q.cn = __fmaf_rn(q.fg, c, q.ig);
        q.tn = tanh_f(q.cn);
        // dc'/dh through the f, i and c gates' pre-activations
        float d = c * (q.fg - q.fg * q.fg) * w[1];
        d = __fmaf_rn(q.g * (q.i - q.i * q.i), w[0], d);
        d = __fmaf_rn(q.i * __fmaf_rn(-q.g, q.g, 1.0f), w[3], d);
        q.dcn_dh = d;
        return q;
    }
    static __device__ __forceinline__ void elem(const float (&p)[G], const float (&w)[G], const float (&sp)[S],
                                                float (&f)[S], float (&A)[S * S], float (&beta)[S]) {
        const float c = sp[0], h = sp[1];
        const Terms q = terms(p, w, c, h);
        const float k = q.o * __fmaf_rn(-q.tn, q.tn, 1.0f);  // dh'/dc'
        f[0] = q.cn;
        f[1] = q.o * q.tn;
        A[0] = q.fg;                                            // dc'/dc
        A[1] = q.dcn_dh;                                        // dc'/dh
        A[2] = k * q.fg;                                        // dh'/dc
        A[3] = __fmaf_rn((q.o - q.o * q.o) * w[2], q.tn, k * q.dcn_dh);  // dh'/dh
        // beta = f - A (c, h): for the c row, c' - f c = i g exactly in real
        // arithmetic, so beta_c = i g - (dc'/dh) h
        beta[0] = __fmaf_rn(-A[1], h, q.ig);
        beta[1] = f[1] - __fmaf_rn(A[2], c, A[3] * h);
    }
    // ---- two channels per instruction (packed f32x2) ----
    struct W2 {
        f2 w0, w1, w2, w3, nw3;
    };
    static __device__ __forceinline__ W2 weights2(const float (&wa)[G], const float (&wb)[G]) {
        return W2{f2{wa[0], wb[0]}, f2{wa[1], wb[1]}, f2{wa[2], wb[2]}, f2{wa[3], wb[3]}, f2{-wa[3], -wb[3]}};
    }
    // warm() on a pair of channels
    static __device__ __forceinline__ void warm2(const f2 (&p)[G], f2 (&f)[S]) {
        const f2 i = sigmoid2(p[0]);
        const f2 o = sigmoid2(p[2]);
        const f2 cn = mul2(i, tanh2(p[3]));
        f[0] = cn;
        f[1] = mul2(o, tanh2(cn));
    }
    // elem() on a pair of channels; sp = (c, h), A row-major (2 x 2)
    static __device__ __forceinline__ void elem2(const f2 (&p)[G], const W2& w, const f2 (&sp)[S], f2 (&f)[S],
                                                 f2 (&A)[S * S], f2 (&beta)[S]) {
        const f2 one = splat2(1.0f), mone = splat2(-1.0f);
        const f2 c = sp[0], h = sp[1];
        const f2 i = sigmoid2(fma2(w.w0, h, p[0]));
        const f2 fg = sigmoid2(add2(fma2(w.w1, h, p[1]), one));
        const f2 o = sigmoid2(fma2(w.w2, h, p[2]));
        const f2 g = tanh2(fma2(w.w3, h, p[3]));
        const f2 ig = mul2(i, g);
        const f2 cn = fma2(fg, c, ig);
        const f2 tn = tanh2(cn);
        // dc'/dh through the f, i and c gates' pre-activations
        f2 d = mul2(mul2(c, fma2(fg, mul2(fg, mone), fg)), w.w1);
        d = fma2(mul2(g, fma2(i, mul2(i, mone), i)), w.w0, d);
        d = fma2(mul2(i, fma2(g, g, mone)), w.nw3, d);  // i (1 - g^2) a_c, both signs flipped
        const f2 k = mul2(mul2(o, fma2(tn, tn, mone)), mone);  // dh'/dc' = o (1 - tn^2)
        f[0] = cn;
        f[1] = mul2(o, tn);
        A[0] = fg;
        A[1] = d;
        A[2] = mul2(k, fg);
        A[3] = fma2(mul2(fma2(o, mul2(o, mone), o), w.w2), tn, mul2(k, d));
        beta[0] = fma2(d, mul2(h, mone), ig);
        beta[1] = sub2(f[1], fma2(A[2], c, mul2(A[3], h)));
    }
    // bwd() on a pair of channels
    static __device__ __forceinline__ void bwd2(const f2 (&p)[G], const W2& w, const f2 (&sp)[S], f2 (&A)[S * S],
                                                f2 (&sens)[NSENS]) {
        const f2 one = splat2(1.0f), mone = splat2(-1.0f);
        const f2 c = sp[0], h = sp[1];
        const f2 i = sigmoid2(fma2(w.w0, h, p[0]));
        const f2 fg = sigmoid2(add2(fma2(w.w1, h, p[1]), one));
        const f2 o = sigmoid2(fma2(w.w2, h, p[2]));
        const f2 g = tanh2(fma2(w.w3, h, p[3]));
        const f2 tn = tanh2(fma2(fg, c, mul2(i, g)));
        const f2 si = mul2(g, fma2(i, mul2(i, mone), i));     // dc'/dp_i = g i (1 - i)
        const f2 sf = mul2(c, fma2(fg, mul2(fg, mone), fg));  // dc'/dp_f = c f (1 - f)
        const f2 nsc = mul2(i, fma2(g, g, mone));             // -(dc'/dp_c) = -i (1 - g^2)
        f2 d = mul2(sf, w.w1);
        d = fma2(si, w.w0, d);
        d = fma2(nsc, w.nw3, d);
        const f2 k = mul2(mul2(o, fma2(tn, tn, mone)), mone);  // dh'/dc' = o (1 - tn^2)
        const f2 dho = mul2(fma2(o, mul2(o, mone), o), tn);    // dh'/dp_o = o (1 - o) tn
        A[0] = fg;
        A[1] = d;
        A[2] = mul2(k, fg);
        A[3] = fma2(dho, w.w2, mul2(k, d));
        sens[0] = si;
        sens[1] = sf;
        sens[2] = mul2(nsc, mone);
        sens[3] = k;
        sens[4] = dho;
        sens[5] = h;
    }
    static __device__ __forceinline__ void grads2(const f2 (&sens)[NSENS], const f2 (&lam)[S], f2 (&dp)[G],
                                                  f2 (&da)[G]) {
        const f2 m = fma2(lam[1], sens[3], lam[0]);
        dp[0] = mul2(m, sens[0]);
        dp[1] = mul2(m, sens[1]);
        dp[2] = mul2(lam[1], sens[4]);
        dp[3] = mul2(m, sens[2]);
#pragma unroll
        for (int g = 0; g < G; ++g) da[g] = mul2(dp[g], sens[5]);
    }
    static __device__ __forceinline__ void bwd(const float (&p)[G], const float (&w)[G], const float (&sp)[S],
                                               float (&A)[S * S], float (&sens)[NSENS]) {
        const float c = sp[0], h = sp[1];
        const Terms q = terms(p, w, c, h);
        const float k = q.o * __fmaf_rn(-q.tn, q.tn, 1.0f);
        const float dho = (q.o - q.o * q.o) * q.tn;
        A[0] = q.fg;
        A[1] = q.dcn_dh;
        A[2] = k * q.fg;
        A[3] = __fmaf_rn(dho, w[2], k * q.dcn_dh);
        sens[0] = q.g * (q.i - q.i * q.i);               // dc'/dp_i
        sens[1] = c * (q.fg - q.fg * q.fg);              // dc'/dp_f
        sens[2] = q.i * __fmaf_rn(-q.g, q.g, 1.0f);      // dc'/dp_c
        sens[3] = k;                                     // dh'/dc'
        sens[4] = dho;                                   // dh'/dp_o
        sens[5] = h;
    }
    static __device__ __forceinline__ void grads(const float (&sens)[NSENS], const float (&lam)[S], float (&dp)[G],
                                                 float (&da)[G]) {
        // lambda . df/dp_g with h' depending on p_i, p_f, p_c only through c'
        const float m = __fmaf_rn(lam[1], sens[3], lam[0]);
        dp[0] = m * sens[0];
        dp[1] = m * sens[1];
        dp[2] = lam[1] * sens[4];
        dp[3] = m * sens[2];
#pragma unroll
        for (int g = 0; g < G; ++g) da[g] = dp[g] * sens[5];
    }
};

// ---- scan element algebra (S = 1 scalar, S = 2 2x2 block) -----------------
// element e = (A, b) acts on a state x as e(x) = A x + b; composition
// (A2, b2) o (A1, b1) = (A2 A1, A2 b1 + b2) applies e1 first.  Every
// application goes through apply(), so the same product is rounded the same
// way wherever it is formed.

template <int S>
struct Elem {
    float A[S * S];
    float b[S];
};

template <int S>
__device__ __forceinline__ void elem_identity(Elem<S>& e) {
#pragma unroll
    for (int i = 0; i < S * S; ++i) e.A[i] = (i % (S + 1) == 0) ? 1.0f : 0.0f;
#pragma unroll
    for (int i = 0; i < S; ++i) e.b[i] = 0.0f;
}

// ---- the same algebra on a pair of channels (packed f32x2) -----------------
// Each operation rounds like its scalar counterpart above, so a pair gives
// the bits two scalar calls would.

// y = A x + b
template <int S>
__device__ __forceinline__ void apply2(const f2 (&A)[S * S], const f2 (&b)[S], const f2 (&x)[S], f2 (&y)[S]) {
    if constexpr (S == 1) {
        y[0] = fma2(A[0], x[0], b[0]);
    } else {
        y[0] = fma2(A[0], x[0], fma2(A[1], x[1], b[0]));
        y[1] = fma2(A[2], x[0], fma2(A[3], x[1], b[1]));
    }
}

// (accA, accb) <- (A, b) o (accA, accb), on pairs
template <int S>
__device__ __forceinline__ void compose_after2(const f2 (&A)[S * S], const f2 (&b)[S], f2 (&accA)[S * S],
                                               f2 (&accb)[S]) {
    if constexpr (S == 1) {
        accb[0] = fma2(A[0], accb[0], b[0]);
        accA[0] = mul2(A[0], accA[0]);
    } else {
        f2 nb[2];
        apply2<2>(A, b, accb, nb);
        f2 nA[4];
        nA[0] = fma2(A[0], accA[0], mul2(A[1], accA[2]));
        nA[1] = fma2(A[0], accA[1], mul2(A[1], accA[3]));
        nA[2] = fma2(A[2], accA[0], mul2(A[3], accA[2]));
        nA[3] = fma2(A[2], accA[1], mul2(A[3], accA[3]));
#pragma unroll
        for (int i = 0; i < 4; ++i) accA[i] = nA[i];
        accb[0] = nb[0];
        accb[1] = nb[1];
    }
}

// y = A x + b
template <int S>
__device__ __forceinline__ void apply(const float (&A)[S * S], const float (&b)[S], const float (&x)[S],
                                      float (&y)[S]) {
    if constexpr (S == 1) {
        y[0] = __fmaf_rn(A[0], x[0], b[0]);
    } else {
        y[0] = __fmaf_rn(A[0], x[0], __fmaf_rn(A[1], x[1], b[0]));
        y[1] = __fmaf_rn(A[2], x[0], __fmaf_rn(A[3], x[1], b[1]));
    }
}

// acc <- e o acc  (e applied after acc)
template <int S>
__device__ __forceinline__ void compose_after(const float (&A)[S * S], const float (&b)[S], Elem<S>& acc) {
    if constexpr (S == 1) {
        acc.b[0] = __fmaf_rn(A[0], acc.b[0], b[0]);
        acc.A[0] = A[0] * acc.A[0];
    } else {
        float nb[2];
        apply<2>(A, b, acc.b, nb);
        float nA[4];
        nA[0] = __fmaf_rn(A[0], acc.A[0], A[1] * acc.A[2]);
        nA[1] = __fmaf_rn(A[0], acc.A[1], A[1] * acc.A[3]);
        nA[2] = __fmaf_rn(A[2], acc.A[0], A[3] * acc.A[2]);
        nA[3] = __fmaf_rn(A[2], acc.A[1], A[3] * acc.A[3]);
#pragma unroll
        for (int i = 0; i < 4; ++i) acc.A[i] = nA[i];
        acc.b[0] = nb[0];
        acc.b[1] = nb[1];
    }
}

}  // namespace pararnn
