// Backward pass of the prefill scan: the gradients of every input and of the initial state,
// given the gradient dy of the output and of the final state.
//
// The forward ("Mamba-3: Improved Sequence Modeling using State Space Principles", Sec. 3.1.1
// Prop. 1, Sec. 3.2.2 Prop. 4, Sec. 3.4, Appendix C) per (batch, head) unit is
//   h_t = a_t h_{t-1} + b_t u_{t-1} + g_t u_t,   u_t = sum_r Bbar_t[r] x_t[r]^T,
//   y_t[r] = h_t^T Cbar_t[r],   Bbar_t = R(Phi_t)^T (norm(B_t) + bias),   Phi_t = Phi_{t-1} + dt_t theta_t.
// With G_t = dL/dh_t = sum_r Cbar_t[r] dy_t[r]^T + a_{t+1} G_{t+1} the gradients split into
// two sweeps that never need h and G at the same token:
//   forward sweep (bwd_fwd_kernel): h_t, hence dCbar_t[r] = h_t dy_t[r] (a contraction over P);
//   reverse sweep (bwd_rev_kernel): G_t, hence du_t = g_t G_t + b_{t+1} G_{t+1},
//     dx_t[r] = du_t^T Bbar_t[r], dBbar_t[r] = du_t x_t[r], db_t = <G_t, u_{t-1}>, dg_t = <G_t, u_t>,
//     and the angle adjoint: Phi_t rotates Bbar_t and Cbar_t, so dPhi_t collects
//     dBbar x Bbar + dCbar x Cbar (the cross product of each pair) and is summed from the end.
// The decay's own gradient needs <G_t, h_{t-1}>, which neither sweep has; it follows instead
// from <G_t, h_t> = dy_t . y_t + a_{t+1} <G_{t+1}, h_t>: with a_t = e^{dt A}, the gradient of
// the log-decay dt_t A_t through the h_{t-1} term is
//   D_t = sum_{s >= t} (dy_s . y_s - b_s db_s - g_s dg_s) + <dL/dh_final, h_final>,
// where dy_s . y_s = sum_r <Cbar_s[r], dCbar_s[r]>. bwd_scalar_kernel takes that suffix sum and
// the chain rule to dt, A and lam (and to the raw projections under the flags);
// bwd_norm_kernel undoes the rotation's partner, the RMS norm, and sums heads that share a
// group's B and C.
//
// Thread layout of the sweeps: one CTA per unit with 2N threads; thread = (pair i, quarter q)
// owns the rows i and i + N/2 (one complex pair, so the rotation is thread-local) and the
// P/4 columns of h or G in registers (16-byte groups interleaved across the quad). Contractions
// over P finish with two shuffles inside the quad; contractions over N with a butterfly across
// the warp's eight pairs and a shared-memory add across warps. A chunk of T tokens is staged in
// shared memory (rotated B and C, x, dy, cos/sin, scalars) before the sequential token loop,
// so the loop has no barrier; the next chunk's global loads (cp.async) fly during the loop.
// bwd_rms_kernel computes the RMS scales of all B and C rows once, before the sweeps.
//
// Summation order: in the sweeps, the cross-warp sums of dx and of the per-token scalar
// partials are shared-memory atomic adds and the B and C bias sums over units are global
// atomic adds, so the sweeps' gradients are not bitwise reproducible run to run (they differ
// in the last bits). The dt_bias sum over units has a fixed order (per-unit shares, then a
// sum over the batch), as every sum of the chunked tensor-core form does.
#include <cuda_bf16.h>

#include "m3_common.cuh"
#include "m3_internal.h"

namespace m3 {
namespace {

constexpr unsigned kFull = 0xffffffffu;

// Asynchronous 16-, 8- and 4-byte global -> shared copies (cp.async); a 16-byte copy with
// valid = false writes zeros and reads nothing.
__device__ __forceinline__ void cp16(void* dst, const void* src, bool valid) {
    const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(d), "l"(src),
                 "r"(valid ? 16 : 0));
}
__device__ __forceinline__ void cp4(void* dst, const void* src) {
    const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(d), "l"(src));
}
__device__ __forceinline__ void cp8(void* dst, const void* src) {
    const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;\n" ::"r"(d), "l"(src));
}

// Two-lane fp32 arithmetic of sm_100 (one packed instruction for two columns):
// fma2 = (a.x b.x + c.x, a.y b.y + c.y), mul2 = (a.x b.x, a.y b.y), round to nearest.
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
    float2 d;
    asm("{.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 dup2(float v) { return make_float2(v, v); }

// Shared-memory layout of one chunk (floats). Slot k = 0..T holds token c0 - 1 + k. RAW holds
// the chunk's inputs as loaded (element size es): B rows (slots 0..T), C, dy and theta rows
// (slots 1..T at k - 1), x rows (0..T), the raw dt, A, lam (slots 1..T at k - 1) and the RMS
// scales of B and C (slots 0..T, per rank).
struct BwdLayout {
    int B, C, X, DY, CS, TH, DC, DB, DX, DTH, SC, SCAL, BIAS, RAW, RDC, RPHI, total;
};
__host__ __device__ inline BwdLayout bwd_layout(int T, int R, int N, int P, int es) {
    BwdLayout l{};
    int o = 0;
    const int S = T + 1;
    l.B = o; o += S * R * N;
    l.C = o; o += S * R * N;
    l.X = o; o += S * R * P;
    l.DY = o; o += S * R * P;
    l.CS = o; o += S * N;         // [k][i] cos, [k][N/2 + i] sin
    l.TH = o; o += S * (N / 2);
    l.DC = o; o += S * R * N;
    l.DB = o; o += S * R * N;
    l.DX = o; o += S * R * P;
    l.DTH = o; o += S * (N / 2);
    l.SC = o; o += (T + 2) * 4;   // per slot: db (from the step before), dg, dy.y, theta.dPhi
    l.SCAL = o; o += S * 8;       // per slot: dt, A, lam, alpha, beta, gamma
    l.BIAS = o; o += 2 * R * N;   // this head's B and C bias (zeros when absent)
    o = (o + 3) / 4 * 4;
    l.RAW = o;
    o += (S * R * N * es + T * R * N * es + S * R * P * es + T * R * P * es +
          T * (N / 2) * es + T * 12 + S * R * 8 + 15) / 16 * 4;
    l.RDC = o; o += T * R * N;    // the reverse sweep's dCbar rows as loaded (slots 1..T)
    l.RPHI = o; o += N / 2;       // the reverse sweep's chunk-start angle as loaded
    l.total = (o + 3) / 4 * 4;
    return l;
}

struct BwdArgs {
    ScanParams f;
    const void* dy;
    const float* dh1;
    const float* dphi1;
    const float* dprevB1;
    const float* dprevx1;
    float* dx;
    float* dB;
    float* dC;
    float* dtheta;
    float* ddt;
    float* dA;
    float* dlam;
    float* dBbias;
    float* dCbias;
    float* ddtbias;
    float* dh0;
    float* dphi0;
    float* dprevB0;
    float* dprevx0;
    float* wdC;    // [b,L,H,R,N] dCbar (forward sweep), then dC after the rotation (reverse)
    float* wdB;    // [b,L,H,R,N] dB after the rotation
    int wd_bf16;   // the chunked form wrote wdB and wdC as bf16 (the norm kernel reads them so)
    float* wphi;   // [units][nchunks][N/2] angle before each chunk
    float* wF;     // [units] <dL/dh_final, h_final>
    float* wsc;    // [units][L][4] db, dg, dy.y, theta.dPhi per token
    float* wprev;  // [units][R][N] gradient of the normalised previous B of the initial state
    float2* wrs;   // [b,L,G,R] RMS scales of B (x) and C (y); null without the norm
    float* wrsp;   // [units][R] RMS scale of the initial state's previous B
    int T;
    int nchunks;
};

// Issues every global load of chunk c (cp.async into the RAW, RDC and RPHI areas) as one
// commit group, without waiting: the loads of the next chunk fly while this one computes.
template <typename T>
__device__ void issue_chunk(const BwdArgs& a, const BwdLayout& lay, float* sm, int64_t u, int c,
                            bool read_dc) {
    constexpr int es = sizeof(T);
    const ScanParams& p = a.f;
    const int N = static_cast<int>(p.N), P = static_cast<int>(p.P), R = static_cast<int>(p.R);
    const int half = N / 2, Tm = a.T;
    const int64_t L = p.L, H = p.H;
    const int64_t bb = u / H, hh = u % H, g = hh / (H / p.G);
    const int tid = threadIdx.x, nth = blockDim.x, warp = tid >> 5, lane = tid & 31;
    const int nwarps = nth >> 5;
    const int rowB = R * N * es, rowX = R * P * es, rowT = half * es;   // bytes
    char* rB = reinterpret_cast<char*>(sm + lay.RAW);
    char* rC = rB + (Tm + 1) * rowB;
    char* rX = rC + Tm * rowB;
    char* rDY = rX + (Tm + 1) * rowX;
    char* rTH = rDY + Tm * rowX;
    float* rS = reinterpret_cast<float*>(rTH + Tm * rowT);

    float2* rRS = reinterpret_cast<float2*>(rS + Tm * 3 + (Tm * 3 & 1));
    const bool norm = a.wrs != nullptr;

    const int64_t c0 = static_cast<int64_t>(c) * Tm;
    const int Tc = static_cast<int>(L - c0 < Tm ? L - c0 : Tm);
    (void)warp; (void)lane; (void)nwarps;
    // ---- one batch of asynchronous loads (region by region; q = j / v by a float
    // reciprocal, exact for these small integers) ----
    const char* Bg = static_cast<const char*>(p.B);
    const char* Cg = static_cast<const char*>(p.C);
    const char* xg = static_cast<const char*>(p.x);
    const char* dyg = static_cast<const char*>(a.dy);
    const char* thg = static_cast<const char*>(p.theta);
    auto divq = [](int j, int v, float inv) { return __float2int_rz((j + 0.5f) * inv); };
    {
        const int vB = rowB / 16;
        const float inv = 1.f / vB;
        for (int j = tid; j < (2 * Tc + 1) * vB; j += nth) {
            int k = divq(j, vB, inv);
            const int o = (j - k * vB) * 16;
            const bool isC = k > Tc;
            if (isC) k -= Tc;     // C: slots 1..Tc
            const int64_t t = c0 - 1 + k;
            const void* src = Bg;
            bool valid = true;
            if (isC) src = Cg + ((bb * L + t) * p.G + g) * rowB + o;
            else if (t >= 0) src = Bg + ((bb * L + t) * p.G + g) * rowB + o;
            else if (p.prevB0) src = static_cast<const char*>(p.prevB0) + u * rowB + o;
            else valid = false;
            cp16(isC ? rC + (k - 1) * rowB + o : rB + k * rowB + o, src, valid);
        }
    }
    {
        const int vX = rowX / 16;
        const float inv = 1.f / vX;
        for (int j = tid; j < (2 * Tc + 1) * vX; j += nth) {
            int k = divq(j, vX, inv);
            const int o = (j - k * vX) * 16;
            const bool isDY = k > Tc;
            if (isDY) k -= Tc;    // dy: slots 1..Tc
            const int64_t t = c0 - 1 + k;
            const void* src = xg;
            bool valid = true;
            if (isDY) src = dyg + ((bb * L + t) * H + hh) * rowX + o;
            else if (t >= 0) src = xg + ((bb * L + t) * H + hh) * rowX + o;
            else if (p.prevx0) src = static_cast<const char*>(p.prevx0) + u * rowX + o;
            else valid = false;
            cp16(isDY ? rDY + (k - 1) * rowX + o : rX + k * rowX + o, src, valid);
        }
    }
    {
        const int vT = rowT / 16;
        const float inv = 1.f / vT;
        for (int j = tid; j < Tc * vT; j += nth) {
            const int k = 1 + divq(j, vT, inv);
            const int o = (j - (k - 1) * vT) * 16;
            cp16(rTH + (k - 1) * rowT + o, thg + ((bb * L + c0 - 1 + k) * H + hh) * rowT + o, true);
        }
    }
    if (read_dc) {
        for (int j = tid; j < half / 4; j += nth)
            cp16(sm + lay.RPHI + 4 * j, a.wphi + (u * a.nchunks + c) * half + 4 * j, true);
        const int vDC = R * N / 4;
        const float inv = 1.f / vDC;
        for (int j = tid; j < Tc * vDC; j += nth) {
            const int k = 1 + divq(j, vDC, inv);
            const int o = (j - (k - 1) * vDC) * 4;
            cp16(sm + lay.RDC + (k - 1) * R * N + o,
                 a.wdC + ((bb * L + c0 - 1 + k) * H + hh) * R * N + o, true);
        }
    }
    for (int e = tid; e < 3 * Tc; e += nth) {
        const int k = 1 + e / 3, w = e - 3 * (e / 3);
        const int64_t si = (bb * L + c0 - 1 + k) * H + hh;
        cp4(rS + (k - 1) * 3 + w, (w == 0 ? p.dt : w == 1 ? p.A : p.lam) + si);
    }
    if (norm) {
        for (int e = tid; e < (Tc + 1) * R; e += nth) {
            const int k = e / R, r = e - k * R;
            const int64_t t = c0 - 1 + k;
            if (t >= 0) cp8(rRS + e, a.wrs + ((bb * L + t) * p.G + g) * R + r);
            else cp4(rRS + e, a.wrsp + u * R + r);
        }
    }
    asm volatile("cp.async.commit_group;\n" ::);
}

// Stages the chunk [c0, c0 + Tc) into shared memory from what issue_chunk loaded: step
// scalars, angles (continuing from phi_start = the angle before token c0; the angle after the
// chunk goes to phi_end when it is set), rotated B (slots 0..Tc) and C (1..Tc), x (0..Tc),
// dy (1..Tc), and the forward sweep's dCbar rows when read_dc. Slot 0 is token c0 - 1: the
// initial state's previous token when c0 = 0.
template <typename T>
__device__ void stage_chunk(const BwdArgs& a, const BwdLayout& lay, float* sm, int64_t u,
                            int64_t c0, int Tc, const float* phi_start, float* phi_end,
                            bool read_dc) {
    constexpr int es = sizeof(T);
    const ScanParams& p = a.f;
    const int N = static_cast<int>(p.N), P = static_cast<int>(p.P), R = static_cast<int>(p.R);
    const int half = N / 2, Tm = a.T;
    const int64_t hh = u % p.H;
    const int tid = threadIdx.x, nth = blockDim.x;
    float* scal = sm + lay.SCAL;
    float* cs = sm + lay.CS;
    const int rowB = R * N * es, rowX = R * P * es, rowT = half * es;   // bytes
    char* rB = reinterpret_cast<char*>(sm + lay.RAW);
    char* rC = rB + (Tm + 1) * rowB;
    char* rX = rC + Tm * rowB;
    char* rDY = rX + (Tm + 1) * rowX;
    char* rTH = rDY + Tm * rowX;
    float* rS = reinterpret_cast<float*>(rTH + Tm * rowT);

    float2* rRS = reinterpret_cast<float2*>(rS + Tm * 3 + (Tm * 3 & 1));
    const bool norm = a.wrs != nullptr;

    auto divq = [](int j, int v, float inv) { return __float2int_rz((j + 0.5f) * inv); };
    asm volatile("cp.async.wait_group 0;\n" ::: "memory");
    __syncthreads();
    if (read_dc) {
        const float4* src = reinterpret_cast<const float4*>(sm + lay.RDC);
        float4* dst = reinterpret_cast<float4*>(sm + lay.DC + R * N);
        for (int e = tid; e < Tc * R * N / 4; e += nth) dst[e] = src[e];
    }

    // ---- step scalars; x, dy and theta to fp32 ----
    const float dtb = p.dt_bias ? p.dt_bias[hh] : 0.f;
    for (int k = 1 + tid; k <= Tc; k += nth) {
        const float d = step_dt(rS[(k - 1) * 3], dtb, p.flags), A = rS[(k - 1) * 3 + 1];
        const float lm = step_lam(rS[(k - 1) * 3 + 2], p.flags);
        const float al = expf(d * A);
        const bool zoh = p.flags & M3_DISC_ZOH;
        float* s = scal + 8 * k;
        s[0] = d; s[1] = A; s[2] = lm; s[3] = al;
        s[4] = zoh ? 0.f : (1.f - lm) * d * al;
        s[5] = zoh ? zoh_gamma(d, A) : lm * d;
    }
    {
        const T* xr = reinterpret_cast<const T*>(rX);
        const T* dyr = reinterpret_cast<const T*>(rDY);
        float* sX = sm + lay.X;
        float* sDY = sm + lay.DY + R * P;
        for (int e = tid; e < (Tc + 1) * R * P; e += nth) sX[e] = to_f(xr[e]);
        for (int e = tid; e < Tc * R * P; e += nth) sDY[e] = to_f(dyr[e]);
        const T* thr = reinterpret_cast<const T*>(rTH);
        float* sTH = sm + lay.TH + half;
        for (int e = tid; e < Tc * half; e += nth) sTH[e] = to_f(thr[e]);
    }
    __syncthreads();

    // ---- angles: the four lanes of a pair's quad walk a quarter of the chunk each, from the
    // chunk-start angle reduced into [-pi, pi], so the hardware sine and cosine stay accurate ----
    {
        const int i = tid >> 2, q = tid & 3;
        const int nk = (Tc + 3) >> 2;
        const int klo = 1 + q * nk, khi = min(Tc, klo + nk - 1);
        const float* th = sm + lay.TH;
        const float ph0 = reduce_2pi(phi_start[i]);
        float loc = 0.f;
        for (int k = klo; k <= khi; ++k) loc = fmaf(scal[8 * k], th[k * half + i], loc);
        const float e1 = __shfl_up_sync(kFull, loc, 1, 4);
        const float e2 = __shfl_up_sync(kFull, loc, 2, 4);
        const float e3 = __shfl_up_sync(kFull, loc, 3, 4);
        float ph = ph0 + ((q >= 1 ? e1 : 0.f) + (q >= 2 ? e2 : 0.f) + (q >= 3 ? e3 : 0.f));
        float sn, cn;
        if (q == 0) {
            __sincosf(ph0, &sn, &cn);
            cs[i] = cn; cs[half + i] = sn;
        }
        for (int k = klo; k <= khi; ++k) {
            ph = fmaf(scal[8 * k], th[k * half + i], ph);
            __sincosf(ph, &sn, &cn);
            cs[k * N + i] = cn; cs[k * N + half + i] = sn;
        }
        if (phi_end && klo <= khi && khi == Tc) phi_end[i] = ph;
    }
    __syncthreads();

    // ---- rotated, normalised, biased B (slots 0..Tc) and C (1..Tc): one thread per pair ----
    {
        const int RH = R * half;
        const float inv = 1.f / RH, invh = 1.f / half;
        const int nBp = (Tc + 1) * RH;
        for (int e = tid; e < nBp + Tc * RH; e += nth) {
            const bool isC = e >= nBp;
            const int j = isC ? e - nBp : e;
            const int kk = divq(j, RH, inv);
            const int rem = j - kk * RH;
            const int r = divq(rem, half, invh), i = rem - r * half;
            const int k = isC ? kk + 1 : kk;
            const T* src = reinterpret_cast<const T*>(isC ? rC + (k - 1) * rowB : rB + k * rowB) + r * N;
            const float* bias = sm + lay.BIAS + (isC ? R * N : 0) + r * N;
            const float scale = norm ? (isC ? rRS[k * R + r].y : rRS[k * R + r].x) : 1.f;
            const float v0 = to_f(src[i]) * scale + bias[i];
            const float v1 = to_f(src[i + half]) * scale + bias[i + half];
            const float c = cs[k * N + i], sn = cs[k * N + half + i];
            float* dst = sm + (isC ? lay.C : lay.B) + (k * R + r) * N;
            dst[i] = v0 * c + v1 * sn;
            dst[i + half] = v1 * c - v0 * sn;
        }
    }
    __syncthreads();
}

// RMS scales of every B and C row (one warp per (b, t, g, r), both vectors) and of the
// initial state's previous B (one warp per (unit, r)): 1 / sqrt(mean(v^2) + eps).
__global__ void __launch_bounds__(256) bwd_rms_kernel(const BwdArgs a, int bf16) {
    const ScanParams& p = a.f;
    const int64_t N = p.N;
    const int lane = threadIdx.x & 31;
    const int64_t item = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nrow = p.b * p.L * p.G * p.R, nprev = p.b * p.H * p.R;
    if (item >= nrow + nprev) return;
    auto ld = [&](const void* base, int64_t off) {
        return bf16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(base)[off])
                    : static_cast<const float*>(base)[off];
    };
    if (item < nrow) {
        float sb = 0.f, sc = 0.f;
        for (int64_t n = lane; n < N; n += 32) {
            const float vb = ld(p.B, item * N + n), vc = ld(p.C, item * N + n);
            sb = fmaf(vb, vb, sb);
            sc = fmaf(vc, vc, sc);
        }
        sb = warp_sum(sb);
        sc = warp_sum(sc);
        if (lane == 0)
            a.wrs[item] = make_float2(rsqrtf(sb / static_cast<float>(N) + p.eps),
                                      rsqrtf(sc / static_cast<float>(N) + p.eps));
    } else {
        const int64_t j = item - nrow;
        float sb = 0.f;
        if (p.prevB0)
            for (int64_t n = lane; n < N; n += 32) {
                const float v = ld(p.prevB0, j * N + n);
                sb = fmaf(v, v, sb);
            }
        sb = warp_sum(sb);
        if (lane == 0) a.wrsp[j] = rsqrtf(sb / static_cast<float>(N) + p.eps);
    }
}

// Loads this head's B and C biases into shared memory (zeros when absent).
__device__ __forceinline__ void load_bias(const BwdArgs& a, const BwdLayout& lay, float* sm,
                                          int64_t hh) {
    const int RN = static_cast<int>(a.f.R * a.f.N);
    for (int e = threadIdx.x; e < 2 * RN; e += blockDim.x) {
        const float* b = e < RN ? a.f.Bbias : a.f.Cbias;
        sm[lay.BIAS + e] = b ? b[hh * RN + (e % RN)] : 0.f;
    }
}

// Column of a thread's e-th register of a row: the quarter q owns the float4 groups
// 16 m + 4 q .. 16 m + 4 q + 3, so the four quarters of a pair read 64 contiguous bytes
// (distinct banks) with one 16-byte load each.
__host__ __device__ __forceinline__ int col_of(int e, int q) { return 16 * (e >> 2) + 4 * q + (e & 3); }

// Sum over the eight lanes of a warp that share the quarter q (lane bits 2..4) of CPQ
// per-column partials, halving the list at each step; the lane then adds its share into the
// shared-memory row of P columns.
template <int CPQ>
__device__ __forceinline__ void add_cols(const float (&v)[CPQ], int lane, float* row) {
    const int q = lane & 3;
    constexpr int n1 = CPQ / 2, n2 = n1 / 2;
    float w1[n1];
    bool up = lane & 16;
#pragma unroll
    for (int j = 0; j < n1; ++j) {
        const float send = up ? v[j] : v[j + n1];
        const float keep = up ? v[j + n1] : v[j];
        w1[j] = keep + __shfl_xor_sync(kFull, send, 16);
    }
    int off = up ? n1 : 0;
    float w2[n2];
    up = lane & 8;
#pragma unroll
    for (int j = 0; j < n2; ++j) {
        const float send = up ? w1[j] : w1[j + n2];
        const float keep = up ? w1[j + n2] : w1[j];
        w2[j] = keep + __shfl_xor_sync(kFull, send, 8);
    }
    off += up ? n2 : 0;
    if constexpr (n2 >= 2) {
        constexpr int n3 = n2 / 2;
        up = lane & 4;
#pragma unroll
        for (int j = 0; j < n3; ++j) {
            const float send = up ? w2[j] : w2[j + n3];
            const float keep = up ? w2[j + n3] : w2[j];
            atomicAdd(row + col_of(off + (up ? n3 : 0) + j, q),
                      keep + __shfl_xor_sync(kFull, send, 4));
        }
    } else {
        const float w = w2[0] + __shfl_xor_sync(kFull, w2[0], 4);
        if (!(lane & 4)) atomicAdd(row + col_of(off, q), w);
    }
}

// Four per-thread partials summed over the warp (halving, then a plain reduction); lanes
// 0, 8, 16, 24 then hold the sums of v0..v3 in some order, returned with its index.
__device__ __forceinline__ float warp_sum4(float v0, float v1, float v2, float v3, int lane,
                                           int* which) {
    bool up = lane & 16;
    const float a0 = (up ? v2 : v0) + __shfl_xor_sync(kFull, up ? v0 : v2, 16);
    const float a1 = (up ? v3 : v1) + __shfl_xor_sync(kFull, up ? v1 : v3, 16);
    int w = up ? 2 : 0;
    up = lane & 8;
    float b = (up ? a1 : a0) + __shfl_xor_sync(kFull, up ? a0 : a1, 8);
    w += up ? 1 : 0;
    b += __shfl_xor_sync(kFull, b, 4);
    b += __shfl_xor_sync(kFull, b, 2);
    b += __shfl_xor_sync(kFull, b, 1);
    *which = w;
    return b;
}

// ---------------------------------------------------------------------------------------
// Forward sweep: h_t token by token; writes dCbar_t = h_t dy_t per token, the angle before
// every chunk and <dL/dh_final, h_final>.
template <typename T, int CPQ, int kThreads>
__global__ void __launch_bounds__(kThreads, kThreads <= 256 ? 2 : 1) bwd_fwd_kernel(const BwdArgs a) {
    extern __shared__ float4 smem4[];
    float* sm = reinterpret_cast<float*>(smem4);
    const ScanParams& p = a.f;
    const int N = static_cast<int>(p.N), P = static_cast<int>(p.P), R = static_cast<int>(p.R);
    const int half = N / 2;
    const int64_t L = p.L, H = p.H;
    const int64_t u = blockIdx.x, bb = u / H, hh = u % H;
    const int tid = threadIdx.x, lane = tid & 31;
    const int i = tid >> 2, q = tid & 3;
    const BwdLayout lay = bwd_layout(a.T, R, N, P, sizeof(T));
    __shared__ float phi_run[128];
    __shared__ float phi_next[128];
    __shared__ float red[32];

    float h0[CPQ], h1[CPQ];
#pragma unroll
    for (int c = 0; c < CPQ; ++c) {
        h0[c] = p.h0 ? p.h0[(u * N + i) * P + col_of(c, q)] : 0.f;
        h1[c] = p.h0 ? p.h0[(u * N + i + half) * P + col_of(c, q)] : 0.f;
    }
    for (int e = tid; e < half; e += blockDim.x) phi_run[e] = p.phi0 ? p.phi0[u * half + e] : 0.f;
    load_bias(a, lay, sm, hh);
    issue_chunk<T>(a, lay, sm, u, 0, false);
    __syncthreads();

    for (int c = 0; c < a.nchunks; ++c) {
        const int64_t c0 = static_cast<int64_t>(c) * a.T;
        const int Tc = static_cast<int>(L - c0 < a.T ? L - c0 : a.T);
        for (int e = tid; e < half; e += blockDim.x)
            a.wphi[(u * a.nchunks + c) * half + e] = phi_run[e];
        stage_chunk<T>(a, lay, sm, u, c0, Tc, phi_run, phi_next, false);
        if (c + 1 < a.nchunks) issue_chunk<T>(a, lay, sm, u, c + 1, false);
        const float* sB = sm + lay.B;
        const float* sX = sm + lay.X;
        const float* sDY = sm + lay.DY;
        float* sDC = sm + lay.DC;
        for (int k = 1; k <= Tc; ++k) {
            const float* s = sm + lay.SCAL + 8 * k;
            const float al = s[3], be = s[4], ga = s[5];
            const float2 al2 = dup2(al);
#pragma unroll
            for (int cc = 0; cc < CPQ; cc += 2) {
                float2 a0 = mul2(al2, make_float2(h0[cc], h0[cc + 1]));
                float2 a1 = mul2(al2, make_float2(h1[cc], h1[cc + 1]));
                h0[cc] = a0.x; h0[cc + 1] = a0.y; h1[cc] = a1.x; h1[cc + 1] = a1.y;
            }
            for (int r = 0; r < R; ++r) {
                const float2 bp0 = dup2(be * sB[((k - 1) * R + r) * N + i]);
                const float2 bp1 = dup2(be * sB[((k - 1) * R + r) * N + i + half]);
                const float2 bc0 = dup2(ga * sB[(k * R + r) * N + i]);
                const float2 bc1 = dup2(ga * sB[(k * R + r) * N + i + half]);
                const float* xp = sX + ((k - 1) * R + r) * P + 4 * q;
                const float* xc = sX + (k * R + r) * P + 4 * q;
#pragma unroll
                for (int cc = 0; cc < CPQ; cc += 4) {
                    const float4 vp = *reinterpret_cast<const float4*>(xp + 4 * cc);
                    const float4 vc = *reinterpret_cast<const float4*>(xc + 4 * cc);
                    const float2 xpv[2] = {make_float2(vp.x, vp.y), make_float2(vp.z, vp.w)};
                    const float2 xcv[2] = {make_float2(vc.x, vc.y), make_float2(vc.z, vc.w)};
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const int e = cc + 2 * j;
                        const float2 n0 = fma2(bp0, xpv[j], fma2(bc0, xcv[j], make_float2(h0[e], h0[e + 1])));
                        const float2 n1 = fma2(bp1, xpv[j], fma2(bc1, xcv[j], make_float2(h1[e], h1[e + 1])));
                        h0[e] = n0.x; h0[e + 1] = n0.y; h1[e] = n1.x; h1[e + 1] = n1.y;
                    }
                }
            }
            for (int r = 0; r < R; ++r) {
                const float* dy = sDY + (k * R + r) * P + 4 * q;
                float2 p0 = make_float2(0.f, 0.f), p1 = make_float2(0.f, 0.f);
#pragma unroll
                for (int cc = 0; cc < CPQ; cc += 4) {
                    const float4 v = *reinterpret_cast<const float4*>(dy + 4 * cc);
                    const float2 v01 = make_float2(v.x, v.y), v23 = make_float2(v.z, v.w);
                    p0 = fma2(make_float2(h0[cc], h0[cc + 1]), v01, p0);
                    p0 = fma2(make_float2(h0[cc + 2], h0[cc + 3]), v23, p0);
                    p1 = fma2(make_float2(h1[cc], h1[cc + 1]), v01, p1);
                    p1 = fma2(make_float2(h1[cc + 2], h1[cc + 3]), v23, p1);
                }
                float d0 = p0.x + p0.y, d1 = p1.x + p1.y;
                d0 += __shfl_xor_sync(kFull, d0, 1);
                d1 += __shfl_xor_sync(kFull, d1, 1);
                d0 += __shfl_xor_sync(kFull, d0, 2);
                d1 += __shfl_xor_sync(kFull, d1, 2);
                if (q == 0) sDC[(k * R + r) * N + i] = d0;
                if (q == 1) sDC[(k * R + r) * N + i + half] = d1;
            }
        }
        __syncthreads();
        // the chunk's angle end, and its dCbar rows out
        for (int e = tid; e < half; e += blockDim.x) phi_run[e] = phi_next[e];
        const int RN4 = R * N / 4;
        for (int e = tid; e < Tc * RN4; e += blockDim.x) {
            const int k = 1 + e / RN4, o = (e % RN4) * 4;
            *reinterpret_cast<float4*>(a.wdC + ((bb * L + c0 - 1 + k) * H + hh) * R * N + o) =
                *reinterpret_cast<const float4*>(sDC + k * R * N + o);
        }
        __syncthreads();
    }
    // <dL/dh_final, h_final>
    float f = 0.f;
    if (a.dh1) {
#pragma unroll
        for (int c = 0; c < CPQ; ++c) {
            f = fmaf(a.dh1[(u * N + i) * P + col_of(c, q)], h0[c], f);
            f = fmaf(a.dh1[(u * N + i + half) * P + col_of(c, q)], h1[c], f);
        }
    }
    f = warp_sum(f);
    if (lane == 0) red[tid >> 5] = f;
    __syncthreads();
    if (tid == 0) {
        float s = 0.f;
        for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) s += red[w];
        a.wF[u] = s;
    }
}

// ---------------------------------------------------------------------------------------
// Reverse sweep: G_t from the end; dx, dtheta, the rotated-back dB and dC per head, the
// per-token partial sums for the scalars, the bias sums and the initial state's gradients.
template <typename T, int CPQ, int kThreads, bool kR1>
__global__ void __launch_bounds__(kThreads, kThreads <= 256 ? 2 : 1) bwd_rev_kernel(const BwdArgs a) {
    extern __shared__ float4 smem4[];
    float* sm = reinterpret_cast<float*>(smem4);
    const ScanParams& p = a.f;
    const int N = static_cast<int>(p.N), P = static_cast<int>(p.P), R = static_cast<int>(p.R);
    const int half = N / 2;
    const int64_t L = p.L, H = p.H;
    const int64_t u = blockIdx.x, bb = u / H, hh = u % H;
    const int tid = threadIdx.x, lane = tid & 31;
    const int i = tid >> 2, q = tid & 3;
    const BwdLayout lay = bwd_layout(a.T, R, N, P, sizeof(T));
    __shared__ float pend[4];

    float G0[CPQ], G1[CPQ];
#pragma unroll
    for (int c = 0; c < CPQ; ++c) {
        G0[c] = a.dh1 ? a.dh1[(u * N + i) * P + col_of(c, q)] : 0.f;
        G1[c] = a.dh1 ? a.dh1[(u * N + i + half) * P + col_of(c, q)] : 0.f;
    }
    float dphi = a.dphi1 ? a.dphi1[u * half + i] : 0.f;
    float a_n = 1.f, b_n = 0.f;         // alpha and beta of the token after the current one
    float accB[2][2] = {{0.f, 0.f}, {0.f, 0.f}}, accC[2][2] = {{0.f, 0.f}, {0.f, 0.f}};

    float* sB = sm + lay.B;
    float* sC = sm + lay.C;
    float* sX = sm + lay.X;
    float* sDY = sm + lay.DY;
    float* sCS = sm + lay.CS;
    float* sTH = sm + lay.TH;
    float* sDC = sm + lay.DC;
    float* sDB = sm + lay.DB;
    float* sDX = sm + lay.DX;
    float* sDTH = sm + lay.DTH;
    float* sSC = sm + lay.SC;

    for (int c = a.nchunks - 1; c >= 0; --c) {
        const int64_t c0 = static_cast<int64_t>(c) * a.T;
        const int Tc = static_cast<int>(L - c0 < a.T ? L - c0 : a.T);
        if (c == a.nchunks - 1) issue_chunk<T>(a, lay, sm, u, c, true);
        for (int e = tid; e < (Tc + 1) * R * P; e += blockDim.x) sDX[e] = 0.f;
        for (int e = tid; e < (a.T + 2) * 4; e += blockDim.x) sSC[e] = 0.f;
        if (c == a.nchunks - 1) load_bias(a, lay, sm, hh);
        __syncthreads();
        stage_chunk<T>(a, lay, sm, u, c0, Tc, sm + lay.RPHI, nullptr, true);
        if (c > 0) issue_chunk<T>(a, lay, sm, u, c - 1, true);

        for (int k = Tc; k >= 1; --k) {
            const float* s = sm + lay.SCAL + 8 * k;
            const float ga = s[5];
            float sg = 0.f, sbn = 0.f, syy = 0.f, dl = 0.f;
            // G_t = a_{t+1} G_{t+1} + sum_r Cbar_t[r] dy_t[r]^T and, per r, the contractions of
            // G_{t+1} (gA) and G_t (gB) with x_t[r] over this thread's columns and the dx partial
            // sum over its rows of Bbar_t[r] du_t, du_t = g_t G_t + b_{t+1} G_{t+1}.
            float gAr[kR1 ? 1 : 8][2], gBr[kR1 ? 1 : 8][2];
            if constexpr (kR1) {
                // one pass from G_{t+1}: du = (g a' + b') G_{t+1} + g Cbar dy^T and
                // G_t x = a' (G_{t+1} x) + Cbar (dy . x)
                const float cb0 = sC[k * N + i], cb1 = sC[k * N + i + half];
                const float bb0 = sB[k * N + i], bb1 = sB[k * N + i + half];
                const float* x = sX + k * P + 4 * q;
                const float* dy = sDY + k * P + 4 * q;
                const float2 coef = dup2(fmaf(ga, a_n, b_n));
                const float2 gs = dup2(ga * fmaf(bb0, cb0, bb1 * cb1));
                const float2 an2 = dup2(a_n), bb0_2 = dup2(bb0), bb1_2 = dup2(bb1);
                const float2 cb0_2 = dup2(cb0), cb1_2 = dup2(cb1);
                float2 gA0 = make_float2(0.f, 0.f), gA1 = gA0, dyx = gA0;
                float v[CPQ];
#pragma unroll
                for (int cc = 0; cc < CPQ; cc += 4) {
                    const float4 xv4 = *reinterpret_cast<const float4*>(x + 4 * cc);
                    const float4 dv4 = *reinterpret_cast<const float4*>(dy + 4 * cc);
                    const float2 xv[2] = {make_float2(xv4.x, xv4.y), make_float2(xv4.z, xv4.w)};
                    const float2 dv[2] = {make_float2(dv4.x, dv4.y), make_float2(dv4.z, dv4.w)};
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const int e = cc + 2 * j;
                        const float2 g0 = make_float2(G0[e], G0[e + 1]);
                        const float2 g1 = make_float2(G1[e], G1[e + 1]);
                        gA0 = fma2(g0, xv[j], gA0);
                        gA1 = fma2(g1, xv[j], gA1);
                        dyx = fma2(dv[j], xv[j], dyx);
                        const float2 w = fma2(coef, fma2(bb0_2, g0, mul2(bb1_2, g1)), mul2(gs, dv[j]));
                        v[e] = w.x; v[e + 1] = w.y;
                        const float2 n0 = fma2(an2, g0, mul2(cb0_2, dv[j]));
                        const float2 n1 = fma2(an2, g1, mul2(cb1_2, dv[j]));
                        G0[e] = n0.x; G0[e + 1] = n0.y; G1[e] = n1.x; G1[e + 1] = n1.y;
                    }
                }
                add_cols<CPQ>(v, lane, sDX + k * P);
                const float sA0 = gA0.x + gA0.y, sA1 = gA1.x + gA1.y, sdx = dyx.x + dyx.y;
                gAr[0][0] = sA0; gAr[0][1] = sA1;
                gBr[0][0] = fmaf(a_n, sA0, cb0 * sdx);
                gBr[0][1] = fmaf(a_n, sA1, cb1 * sdx);
            } else {
                float go0[CPQ], go1[CPQ];
#pragma unroll
                for (int cc = 0; cc < CPQ; ++cc) {
                    go0[cc] = G0[cc]; go1[cc] = G1[cc];
                    G0[cc] *= a_n; G1[cc] *= a_n;
                }
                for (int r = 0; r < R; ++r) {
                    const float cb0 = sC[(k * R + r) * N + i], cb1 = sC[(k * R + r) * N + i + half];
                    const float* dy = sDY + (k * R + r) * P + 4 * q;
#pragma unroll
                    for (int cc = 0; cc < CPQ; cc += 4) {
                        const float4 v = *reinterpret_cast<const float4*>(dy + 4 * cc);
                        const float dv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            G0[cc + j] = fmaf(cb0, dv[j], G0[cc + j]);
                            G1[cc + j] = fmaf(cb1, dv[j], G1[cc + j]);
                        }
                    }
                }
                for (int r = 0; r < R; ++r) {
                    const float bb0 = sB[(k * R + r) * N + i], bb1 = sB[(k * R + r) * N + i + half];
                    const float* x = sX + (k * R + r) * P + 4 * q;
                    float gA0 = 0.f, gA1 = 0.f, gB0 = 0.f, gB1 = 0.f;
                    float v[CPQ];
#pragma unroll
                    for (int cc = 0; cc < CPQ; cc += 4) {
                        const float4 xv4 = *reinterpret_cast<const float4*>(x + 4 * cc);
                        const float xv[4] = {xv4.x, xv4.y, xv4.z, xv4.w};
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const int e = cc + j;
                            gA0 = fmaf(go0[e], xv[j], gA0); gA1 = fmaf(go1[e], xv[j], gA1);
                            gB0 = fmaf(G0[e], xv[j], gB0); gB1 = fmaf(G1[e], xv[j], gB1);
                            v[e] = ga * fmaf(bb0, G0[e], bb1 * G1[e]) + b_n * fmaf(bb0, go0[e], bb1 * go1[e]);
                        }
                    }
                    add_cols<CPQ>(v, lane, sDX + (k * R + r) * P);
                    gAr[r][0] = gA0; gAr[r][1] = gA1; gBr[r][0] = gB0; gBr[r][1] = gB1;
                }
            }
            for (int r = 0; r < (kR1 ? 1 : R); ++r) {
                const float bb0 = sB[(k * R + r) * N + i], bb1 = sB[(k * R + r) * N + i + half];
                const float gA0 = gAr[r][0], gA1 = gAr[r][1], gB0 = gBr[r][0], gB1 = gBr[r][1];
                sg = fmaf(bb0, gB0, fmaf(bb1, gB1, sg));
                sbn = fmaf(bb0, gA0, fmaf(bb1, gA1, sbn));
                float db0 = fmaf(ga, gB0, b_n * gA0), db1 = fmaf(ga, gB1, b_n * gA1);
                db0 += __shfl_xor_sync(kFull, db0, 1);
                db1 += __shfl_xor_sync(kFull, db1, 1);
                db0 += __shfl_xor_sync(kFull, db0, 2);
                db1 += __shfl_xor_sync(kFull, db1, 2);
                if (kR1) {
                    // B on lane 0 and C on lane 1 of the quad
                    const float co = sCS[k * N + i], si = sCS[k * N + half + i];
                    if (q == 0) {
                        dl += db0 * bb1 - db1 * bb0;
                        const float nB0 = db0 * co - db1 * si, nB1 = db0 * si + db1 * co;
                        sDB[k * N + i] = nB0;
                        sDB[k * N + i + half] = nB1;
                        accB[0][0] += nB0; accB[0][1] += nB1;
                    } else if (q == 1) {
                        const float cb0 = sC[k * N + i], cb1 = sC[k * N + i + half];
                        float* dcp = sDC + k * N;
                        const float dc0 = dcp[i], dc1 = dcp[i + half];
                        dl += dc0 * cb1 - dc1 * cb0;
                        syy = fmaf(cb0, dc0, fmaf(cb1, dc1, syy));
                        const float nC0 = dc0 * co - dc1 * si, nC1 = dc0 * si + dc1 * co;
                        dcp[i] = nC0;
                        dcp[i + half] = nC1;
                        accC[0][0] += nC0; accC[0][1] += nC1;
                    }
                } else if (q == (r & 3)) {
                    const float cb0 = sC[(k * R + r) * N + i], cb1 = sC[(k * R + r) * N + i + half];
                    float* dcp = sDC + (k * R + r) * N;
                    const float dc0 = dcp[i], dc1 = dcp[i + half];
                    const float co = sCS[k * N + i], si = sCS[k * N + half + i];
                    dl += db0 * bb1 - db1 * bb0 + dc0 * cb1 - dc1 * cb0;
                    syy = fmaf(cb0, dc0, fmaf(cb1, dc1, syy));
                    const float nB0 = db0 * co - db1 * si, nB1 = db0 * si + db1 * co;
                    const float nC0 = dc0 * co - dc1 * si, nC1 = dc0 * si + dc1 * co;
                    sDB[(k * R + r) * N + i] = nB0;
                    sDB[(k * R + r) * N + i + half] = nB1;
                    dcp[i] = nC0;
                    dcp[i + half] = nC1;
                    accB[r >> 2][0] += nB0; accB[r >> 2][1] += nB1;
                    accC[r >> 2][0] += nC0; accC[r >> 2][1] += nC1;
                }
            }
            dl += __shfl_xor_sync(kFull, dl, 1);
            dl += __shfl_xor_sync(kFull, dl, 2);
            dphi += dl;
            float thd = 0.f;
            if (q == 0) {
                sDTH[k * half + i] = s[0] * dphi;
                thd = sTH[k * half + i] * dphi;
            }
            int which;
            const float w = warp_sum4(sbn, sg, syy, thd, lane, &which);
            if ((lane & 7) == 0) {
                // which: 0 = db of the next token, 1 = dg, 2 = dy.y, 3 = theta.dPhi
                if (which == 0) atomicAdd(sSC + (k + 1) * 4 + 0, w);
                else atomicAdd(sSC + k * 4 + which, w);
            }
            a_n = s[3];
            b_n = s[4];
        }

        if (c == 0) {
            // token -1: the initial state's h, previous token and angle
            if (a.dh0) {
#pragma unroll
                for (int cc = 0; cc < CPQ; ++cc) {
                    a.dh0[(u * N + i) * P + col_of(cc, q)] = a_n * G0[cc];
                    a.dh0[(u * N + i + half) * P + col_of(cc, q)] = a_n * G1[cc];
                }
            }
            float sbn = 0.f, dl = 0.f;
            for (int r = 0; r < R; ++r) {
                const float bb0 = sB[r * N + i], bb1 = sB[r * N + i + half];
                const float* x = sX + r * P;
                float gA0 = 0.f, gA1 = 0.f;
                float v[CPQ];
#pragma unroll
                for (int e = 0; e < CPQ; ++e) {
                    const float xe = x[col_of(e, q)];
                    gA0 = fmaf(G0[e], xe, gA0);
                    gA1 = fmaf(G1[e], xe, gA1);
                    v[e] = b_n * fmaf(bb0, G0[e], bb1 * G1[e]);
                }
                add_cols<CPQ>(v, lane, sDX + r * P);
                sbn = fmaf(bb0, gA0, fmaf(bb1, gA1, sbn));
                float db0 = b_n * gA0, db1 = b_n * gA1;
                db0 += __shfl_xor_sync(kFull, db0, 1);
                db1 += __shfl_xor_sync(kFull, db1, 1);
                db0 += __shfl_xor_sync(kFull, db0, 2);
                db1 += __shfl_xor_sync(kFull, db1, 2);
                if (q == (r & 3)) {
                    const float co = sCS[i], si = sCS[half + i];
                    dl += db0 * bb1 - db1 * bb0;
                    const float nB0 = db0 * co - db1 * si, nB1 = db0 * si + db1 * co;
                    sDB[r * N + i] = nB0;
                    sDB[r * N + i + half] = nB1;
                    accB[r >> 2][0] += nB0; accB[r >> 2][1] += nB1;
                }
            }
            dl += __shfl_xor_sync(kFull, dl, 1);
            dl += __shfl_xor_sync(kFull, dl, 2);
            if (q == 0 && a.dphi0) a.dphi0[u * half + i] = dphi + dl;
            int which;
            const float w = warp_sum4(sbn, 0.f, 0.f, 0.f, lane, &which);
            if ((lane & 7) == 0 && which == 0) atomicAdd(sSC + 4, w);
        }
        __syncthreads();

        // chunk out: dx, dtheta, dB and dC per head, the scalar partials
        const int RP4 = R * P / 4;
        for (int e = tid; e < Tc * RP4; e += blockDim.x) {
            const int k = 1 + e / RP4, o = (e % RP4) * 4;
            const int64_t t = c0 - 1 + k;
            float4 v = *reinterpret_cast<const float4*>(sDX + k * R * P + o);
            if (t == L - 1 && a.dprevx1) {
                const float4 w = *reinterpret_cast<const float4*>(a.dprevx1 + u * R * P + o);
                v.x += w.x; v.y += w.y; v.z += w.z; v.w += w.w;
            }
            *reinterpret_cast<float4*>(a.dx + ((bb * L + t) * H + hh) * R * P + o) = v;
        }
        const int h4 = half / 4;
        for (int e = tid; e < Tc * h4; e += blockDim.x) {
            const int k = 1 + e / h4, o = (e % h4) * 4;
            *reinterpret_cast<float4*>(a.dtheta + ((bb * L + c0 - 1 + k) * H + hh) * half + o) =
                *reinterpret_cast<const float4*>(sDTH + k * half + o);
        }
        const int RN4 = R * N / 4;
        for (int e = tid; e < Tc * RN4; e += blockDim.x) {
            const int k = 1 + e / RN4, o = (e % RN4) * 4;
            const int64_t off = ((bb * L + c0 - 1 + k) * H + hh) * R * N + o;
            *reinterpret_cast<float4*>(a.wdB + off) = *reinterpret_cast<const float4*>(sDB + k * R * N + o);
            *reinterpret_cast<float4*>(a.wdC + off) = *reinterpret_cast<const float4*>(sDC + k * R * N + o);
        }
        float* wsc = a.wsc + u * L * 4;
        for (int e = tid; e < (Tc - 1) * 4; e += blockDim.x) {
            const int k = 2 + e / 4, j = e % 4;
            wsc[(c0 - 1 + k) * 4 + j] = sSC[k * 4 + j];
        }
        if (tid < 4) {
            // the token after this chunk got its db from this chunk's last step
            if (c0 + Tc < L) wsc[(c0 + Tc) * 4 + tid] = pend[tid] + (tid == 0 ? sSC[(Tc + 1) * 4] : 0.f);
            pend[tid] = sSC[4 + tid];
            if (c == 0) wsc[tid] = sSC[4 + tid];
        }
        if (c == 0) {
            for (int e = tid; e < RP4; e += blockDim.x)
                if (a.dprevx0)
                    *reinterpret_cast<float4*>(a.dprevx0 + u * R * P + e * 4) =
                        *reinterpret_cast<const float4*>(sDX + e * 4);
            for (int e = tid; e < RN4; e += blockDim.x)
                *reinterpret_cast<float4*>(a.wprev + u * R * N + e * 4) =
                    *reinterpret_cast<const float4*>(sDB + e * 4);
        }
        __syncthreads();
    }
    // the biases: each unit adds its sums over the sequence
    if (kR1) {
        if (q == 0 && a.dBbias) {
            atomicAdd(a.dBbias + hh * N + i, accB[0][0]);
            atomicAdd(a.dBbias + hh * N + i + half, accB[0][1]);
        }
        if (q == 1 && a.dCbias) {
            atomicAdd(a.dCbias + hh * N + i, accC[0][0]);
            atomicAdd(a.dCbias + hh * N + i + half, accC[0][1]);
        }
    } else {
        for (int rr = 0; rr < 2; ++rr) {
            const int r = q + 4 * rr;
            if (r >= R) break;
            if (a.dBbias) {
                atomicAdd(a.dBbias + (hh * R + r) * N + i, accB[rr][0]);
                atomicAdd(a.dBbias + (hh * R + r) * N + i + half, accB[rr][1]);
            }
            if (a.dCbias) {
                atomicAdd(a.dCbias + (hh * R + r) * N + i, accC[rr][0]);
                atomicAdd(a.dCbias + (hh * R + r) * N + i + half, accC[rr][1]);
            }
        }
    }
}

// ---------------------------------------------------------------------------------------
// Step scalars: the suffix sum D_t and the chain rule to dt, A, lam (and the raw
// projections). One CTA per unit walks the sequence from the end in tiles.
constexpr int kScalThreads = 256, kScalPer = 4;

__global__ void __launch_bounds__(kScalThreads) bwd_scalar_kernel(const BwdArgs a) {
    const ScanParams& p = a.f;
    const int64_t L = p.L, H = p.H;
    const int64_t u = blockIdx.x, bb = u / H, hh = u % H;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    __shared__ float wtot[kScalThreads / 32];
    __shared__ float red[kScalThreads / 32];
    const float* wsc = a.wsc + u * L * 4;
    const float dtb = p.dt_bias ? p.dt_bias[hh] : 0.f;
    const bool zoh = p.flags & M3_DISC_ZOH;
    float carry = a.wF[u];
    float bias_sum = 0.f;
    constexpr int kTile = kScalThreads * kScalPer;
    for (int64_t t_end = L; t_end > 0; t_end -= kTile) {
        const int64_t t0 = t_end - kTile;   // may be negative: those tokens are skipped
        const int blk = kScalThreads - 1 - tid;   // thread 0 takes the last block of the tile
        float e[kScalPer];
        float tot = 0.f;
#pragma unroll
        for (int j = 0; j < kScalPer; ++j) {
            const int64_t t = t0 + blk * kScalPer + j;
            e[j] = 0.f;
            if (t >= 0) {
                const int64_t si = (bb * L + t) * H + hh;
                const float d = step_dt(p.dt[si], dtb, p.flags), A = p.A[si];
                const float lm = step_lam(p.lam[si], p.flags);
                const float al = expf(d * A);
                const float be = zoh ? 0.f : (1.f - lm) * d * al;
                const float ga = zoh ? zoh_gamma(d, A) : lm * d;
                e[j] = wsc[t * 4 + 2] - be * wsc[t * 4 + 0] - ga * wsc[t * 4 + 1];
            }
            tot += e[j];
        }
        // suffix sums over blocks: an inclusive prefix over tid (blocks in reverse order)
        float incl = warp_inclusive_scan(tot);
        if (lane == 31) wtot[warp] = incl;
        __syncthreads();
        float before = 0.f;
        for (int w = 0; w < warp; ++w) before += wtot[w];
        float tile_sum = 0.f;
        for (int w = 0; w < kScalThreads / 32; ++w) tile_sum += wtot[w];
        float D = carry + before + incl - tot;   // everything after this block
        for (int j = kScalPer - 1; j >= 0; --j) {
            const int64_t t = t0 + blk * kScalPer + j;
            D += e[j];
            if (t < 0) continue;
            const int64_t si = (bb * L + t) * H + hh;
            const float draw = p.dt[si], A = p.A[si], lraw = p.lam[si];
            const float d = step_dt(draw, dtb, p.flags), lm = step_lam(lraw, p.flags);
            const float al = expf(d * A);
            const float db = wsc[t * 4 + 0], dg = wsc[t * 4 + 1], thd = wsc[t * 4 + 3];
            float gdt, gA, glam;
            if (zoh) {
                // gamma = (e^{dA} - 1) / A: d gamma / d dt = alpha, d gamma / d A = (dt alpha - gamma) / A,
                // by its series dt^2 (1/2 + x/3 + x^2/8 + x^3/30 + x^4/144) for small x = dt A
                const float x = d * A;
                const float dgdA = fabsf(x) < 0.05f
                    ? d * d * (0.5f + x * (1.f / 3.f + x * (0.125f + x * (1.f / 30.f + x * (1.f / 144.f)))))
                    : (d * al - zoh_gamma(d, A)) / A;
                gdt = D * A + dg * al + thd;
                gA = D * d + dg * dgdA;
                glam = 0.f;
            } else {
                gdt = D * A + db * (1.f - lm) * al * fmaf(d, A, 1.f) + dg * lm + thd;
                gA = D * d + db * (1.f - lm) * d * d * al;
                glam = (dg - db * al) * d;
            }
            if (p.flags & M3_DT_SOFTPLUS) {
                const float v = draw + dtb;
                gdt *= __frcp_rn(1.f + __expf(-v));   // softplus' = sigmoid
                bias_sum += gdt;
            }
            if (p.flags & M3_LAM_SIGMOID) glam *= lm * (1.f - lm);
            a.ddt[si] = gdt;
            a.dA[si] = gA;
            a.dlam[si] = glam;
        }
        carry += tile_sum;
        __syncthreads();
    }
    if (a.ddtbias && (p.flags & M3_DT_SOFTPLUS)) {
        bias_sum = warp_sum(bias_sum);
        if (lane == 0) red[warp] = bias_sum;
        __syncthreads();
        if (tid == 0) {
            float s = 0.f;
            for (int w = 0; w < kScalThreads / 32; ++w) s += red[w];
            a.wphi[u] = s;   // this unit's share; bwd_dtbias_kernel sums the batch in order
        }
    }
}

// dt_bias[h] = sum over the batch of the units' shares, in a fixed order (the per-chunk angle
// buffer, no longer needed, holds the shares).
__global__ void __launch_bounds__(256) bwd_dtbias_kernel(const float* __restrict__ share,
                                                         int64_t b, int64_t H, float* ddtbias) {
    const int64_t h = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (h >= H) return;
    float v = 0.f;
    for (int64_t i = 0; i < b; ++i) v += share[i * H + h];
    ddtbias[h] = v;
}

// ---------------------------------------------------------------------------------------
// RMS-norm backward and the sum over the heads of a group: one warp per (token, group, r,
// B or C), plus one per (unit, r) for the initial state's previous B (per head).
__global__ void __launch_bounds__(256) bwd_norm_kernel(const BwdArgs a, int bf16) {
    const ScanParams& p = a.f;
    const int64_t L = p.L, H = p.H, Gn = p.G, N = p.N, R = p.R;
    const int64_t hpg = H / Gn;
    const int lane = threadIdx.x & 31;
    const int64_t item = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t ntok = p.b * L * Gn * R * 2, nprev = p.b * H * R;
    if (item >= ntok + nprev) return;
    auto raw = [&](const void* base, int64_t off) {
        return bf16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(base)[off])
                    : static_cast<const float*>(base)[off];
    };
    const void* src;
    int64_t src_off;
    float* dst;
    const float* extra = nullptr;   // final state's prev_B gradient, summed over the group
    int64_t h_first = 0, nh = 0, dn_stride = 0, dn_off = 0;
    const float* dn_base;
    bool dn_h = false;   // the per-head rows are bf16
    if (item < ntok) {
        const int isC = static_cast<int>(item & 1);
        const int64_t rest = item >> 1;
        const int64_t r = rest % R, g = (rest / R) % Gn, tok = rest / (R * Gn);   // tok = b*L + t
        const int64_t bb = tok / L, t = tok % L;
        src = isC ? p.C : p.B;
        src_off = ((tok * Gn + g) * R + r) * N;
        dst = (isC ? a.dC : a.dB) + src_off;
        h_first = g * hpg;
        nh = hpg;
        dn_off = ((tok * H + h_first) * R + r) * N;
        dn_base = isC ? a.wdC : a.wdB;
        dn_h = a.wd_bf16 != 0;
        dn_stride = R * N;
        if (!isC && t == L - 1 && a.dprevB1) extra = a.dprevB1 + ((bb * H + h_first) * R + r) * N;
    } else {
        const int64_t j = item - ntok;   // (unit, r)
        if (!a.dprevB0) return;
        src = p.prevB0;
        src_off = j * N;
        dst = a.dprevB0 + j * N;
        nh = 1;
        dn_base = a.wprev;
        dn_off = j * N;
        dn_stride = 0;
    }
    // N <= 256: at most eight elements per lane, kept in registers
    float dnv[8], vv[8];
    float ss = 0.f, dot = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int64_t n = lane + 32 * j;
        dnv[j] = 0.f;
        vv[j] = 0.f;
        if (n < N) {
            if (dn_h) {
                // the group's heads in order, eight loads in flight
                const __nv_bfloat16* hb = reinterpret_cast<const __nv_bfloat16*>(dn_base) + dn_off;
#pragma unroll 8
                for (int64_t h = 0; h < nh; ++h) dnv[j] += __bfloat162float(hb[h * dn_stride + n]);
            } else {
                for (int64_t h = 0; h < nh; ++h) dnv[j] += dn_base[dn_off + h * dn_stride + n];
            }
            vv[j] = src ? raw(src, src_off + n) : 0.f;
            ss = fmaf(vv[j], vv[j], ss);
            dot = fmaf(vv[j], dnv[j], dot);
        }
    }
    ss = warp_sum(ss);
    dot = warp_sum(dot);
    const float s = p.bc_norm ? rsqrtf(ss / static_cast<float>(N) + p.eps) : 1.f;
    const float k = p.bc_norm ? s * s * s / static_cast<float>(N) * dot : 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int64_t n = lane + 32 * j;
        if (n >= N) break;
        float o = s * dnv[j] - k * vv[j];
        if (extra)
            for (int64_t h = 0; h < nh; ++h) o += extra[h * R * N + n];
        dst[n] = o;
    }
}

template <typename T, int CPQ, int kThreads>
cudaError_t launch_sweeps(const BwdArgs& a, size_t smem, cudaStream_t s) {
    const int units = static_cast<int>(a.f.b * a.f.H);
    const int threads = static_cast<int>(2 * a.f.N);
    auto kf = bwd_fwd_kernel<T, CPQ, kThreads>;
    auto kr = a.f.R == 1 ? bwd_rev_kernel<T, CPQ, kThreads, true>
                         : bwd_rev_kernel<T, CPQ, kThreads, false>;
    cudaError_t e = cudaFuncSetAttribute(kf, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kr, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    kf<<<units, threads, smem, s>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    kr<<<units, threads, smem, s>>>(a);
    return cudaGetLastError();
}

template <typename T, int kThreads>
cudaError_t launch_sweeps_p(const BwdArgs& a, size_t smem, cudaStream_t s) {
    switch (a.f.P) {
        case 16: return launch_sweeps<T, 4, kThreads>(a, smem, s);
        case 32: return launch_sweeps<T, 8, kThreads>(a, smem, s);
        case 64: return launch_sweeps<T, 16, kThreads>(a, smem, s);
        default: return launch_sweeps<T, 32, kThreads>(a, smem, s);
    }
}

}  // namespace

int bwd_chunk_tokens(int64_t R) { return static_cast<int>(R >= 16 ? 1 : 16 / R); }

size_t scan_bwd_workspace_floats(int64_t b, int64_t L, int64_t H, int64_t N, int64_t R) {
    const int64_t T = bwd_chunk_tokens(R), nch = (L + T - 1) / T, units = b * H;
    auto r64 = [](int64_t v) { return (v + 63) / 64 * 64; };   // 256-byte regions
    return static_cast<size_t>(2 * r64(b * L * H * R * N) + r64(units * nch * (N / 2)) +
                               r64(units) + r64(units * L * 4) + r64(units * R * N) +
                               r64(2 * b * L * H * R) + r64(units * R));
}

cudaError_t launch_scan_bwd(const ScanParams& f, const BwdGrads& g, bool bf16, float* ws,
                            void* tc_ws, int32_t* status, cudaStream_t s) {
    BwdArgs a{};
    a.f = f;
    a.dy = g.dy;
    a.dh1 = g.dh1; a.dphi1 = g.dphi1; a.dprevB1 = g.dprevB1; a.dprevx1 = g.dprevx1;
    a.dx = g.dx; a.dB = g.dB; a.dC = g.dC; a.dtheta = g.dtheta;
    a.ddt = g.ddt; a.dA = g.dA; a.dlam = g.dlam;
    a.dBbias = g.dBbias; a.dCbias = g.dCbias; a.ddtbias = g.ddtbias;
    a.dh0 = g.dh0; a.dphi0 = g.dphi0; a.dprevB0 = g.dprevB0; a.dprevx0 = g.dprevx0;
    a.T = bwd_chunk_tokens(f.R);
    a.nchunks = static_cast<int>((f.L + a.T - 1) / a.T);
    const int64_t units = f.b * f.H, nch = a.nchunks;
    auto r64 = [](int64_t v) { return (v + 63) / 64 * 64; };
    float* o = ws;
    a.wdC = o; o += r64(f.b * f.L * f.H * f.R * f.N);
    a.wdB = o; o += r64(f.b * f.L * f.H * f.R * f.N);
    a.wphi = o; o += r64(units * nch * (f.N / 2));
    a.wF = o; o += r64(units);
    a.wsc = o; o += r64(units * f.L * 4);
    a.wprev = o; o += r64(units * f.R * f.N);
    if (f.bc_norm) {
        a.wrs = reinterpret_cast<float2*>(o);   // G <= H rows: the [b,L,H,R] region holds them
        o += r64(2 * f.b * f.L * f.H * f.R);
        a.wrsp = o;
    }

    cudaError_t e;
    if (a.ddtbias && (e = cudaMemsetAsync(a.ddtbias, 0, sizeof(float) * f.H, s)) != cudaSuccess) return e;
    if (tc_ws) {
        // the chunked tensor-core form writes dx, dtheta, the initial state's h, phi and
        // prev_x gradients, the bias gradients and the intermediate buffers of the two kernels
        // below in place of the sweeps
        BwdTcOut o{};
        o.dy = g.dy;
        o.dh1 = g.dh1; o.dphi1 = g.dphi1; o.dprevx1 = g.dprevx1;
        o.dx = g.dx; o.dtheta = g.dtheta;
        o.wdB = a.wdB; o.wdC = a.wdC; o.wsc = a.wsc; o.wprev = a.wprev; o.wF = a.wF;
        a.wd_bf16 = 1;
        o.dh0 = g.dh0; o.dphi0 = g.dphi0; o.dprevx0 = g.dprevx0;
        o.dBbias = g.dBbias; o.dCbias = g.dCbias;
        o.status = status;
        if ((e = launch_bwd_tc(f, o, tc_ws, s)) != cudaSuccess) return e;
    } else {
        if (a.dBbias && (e = cudaMemsetAsync(a.dBbias, 0, sizeof(float) * f.H * f.R * f.N, s)) != cudaSuccess) return e;
        if (a.dCbias && (e = cudaMemsetAsync(a.dCbias, 0, sizeof(float) * f.H * f.R * f.N, s)) != cudaSuccess) return e;
        const BwdLayout lay = bwd_layout(a.T, static_cast<int>(f.R), static_cast<int>(f.N),
                                         static_cast<int>(f.P), bf16 ? 2 : 4);
        const size_t smem = sizeof(float) * lay.total;
        if (f.bc_norm) {
            const int64_t items = f.b * f.L * f.G * f.R + units * f.R;
            bwd_rms_kernel<<<static_cast<unsigned>((items * 32 + 255) / 256), 256, 0, s>>>(a, bf16 ? 1 : 0);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
        }
        if (f.N <= 128)
            e = bf16 ? launch_sweeps_p<__nv_bfloat16, 256>(a, smem, s)
                     : launch_sweeps_p<float, 256>(a, smem, s);
        else
            e = bf16 ? launch_sweeps_p<__nv_bfloat16, 512>(a, smem, s)
                     : launch_sweeps_p<float, 512>(a, smem, s);
        if (e != cudaSuccess) return e;
    }
    bwd_scalar_kernel<<<static_cast<unsigned>(units), kScalThreads, 0, s>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (a.ddtbias && (f.flags & M3_DT_SOFTPLUS)) {
        bwd_dtbias_kernel<<<static_cast<unsigned>((f.H + 255) / 256), 256, 0, s>>>(a.wphi, f.b, f.H,
                                                                                  a.ddtbias);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    const int64_t items = f.b * f.L * f.G * f.R * 2 + units * f.R;
    const int64_t blocks = (items * 32 + 255) / 256;
    bwd_norm_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(a, bf16 ? 1 : 0);
    return cudaGetLastError();
}

size_t scan_bwd_smem_bytes(int64_t N, int64_t P, int64_t R) {
    const BwdLayout lay = bwd_layout(bwd_chunk_tokens(R), static_cast<int>(R),
                                     static_cast<int>(N), static_cast<int>(P), 4);
    return sizeof(float) * lay.total;
}

}  // namespace m3
