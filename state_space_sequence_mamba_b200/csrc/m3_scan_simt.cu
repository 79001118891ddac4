// Chunked prefill scan on CUDA cores (FP32 FMA throughout, no tensor cores).
//
// This is the exact-arithmetic instantiation: fp32 inputs keep full fp32 precision, which the
// TF32/bf16 tensor-core path cannot. It also runs any supported shape the tensor-core kernel
// is not specialised for. One CTA owns one (batch, head) unit and walks its chunks in order,
// with the N x P fp32 state resident in shared memory.
//
// The chunked form ("Mamba-3: Improved Sequence Modeling using State Space Principles",
// Sec. 3.1.3 eq. 7 for the L = L1 . L2 mask, Sec. 3.3 for the chunked algorithm and MIMO,
// Appendix B.3 for the rotated frame) carries the primed state
//     h'_t = h~_t + (1 - lam_{t+1}) dt_{t+1} v_t,        v_t = sum_r Bbar_t[r] x_t[r]^T,
// which obeys h'_t = alpha_t h'_{t-1} + w_t v_t with w_t = gamma_t + (1 - lam_{t+1}) dt_{t+1}
// (w = gamma for the last token of the sequence). For a chunk starting from H0 = h'_{start-1}:
//     Y   = (Cbar Bbar^T o M) X + diag(e^{cum}) Cbar H0,
//           M[t,s] = e^{cum_t - cum_s} w_s (s < t), gamma_t (s = t), 0 (s > t),
//     H1  = e^{cum_end} H0 + Bbar^T diag(e^{cum_end - cum_s} w_s) X,
// where cum is the chunk-local inclusive sum of dt*A. MIMO rows are (token, rank) pairs and
// the token mask is expanded by a full R x R block. A stored initial state enters as
// h'_{-1} = h~_{-1} + (1 - lam_0) dt_0 Bbar_{-1} x_{-1}^T.
#include "m3_common.cuh"
#include "m3_internal.h"

namespace m3 {

namespace {

constexpr int kSimtThreads = 256;

struct SimtLayout {
    int64_t H, Bb, Cb, X, S, phi, rsB, rsC, sc;  // float offsets
    int64_t total;                               // floats
};

__host__ __device__ inline SimtLayout simt_layout(int64_t N, int64_t P, int64_t Q, int64_t R) {
    SimtLayout l;
    const int64_t QR = Q * R;
    int64_t o = 0;
    l.H = o; o += N * P;
    l.Bb = o; o += QR * N;
    l.Cb = o; o += QR * N;
    l.X = o; o += QR * P;
    l.S = o; o += QR * QR;
    l.phi = o; o += N / 2;
    l.rsB = o; o += QR + R;  // + R for the stored previous B
    l.rsC = o; o += QR;
    l.sc = o; o += 8 * (Q + 1);
    l.total = o;
    return l;
}

// sc block: per token t of the chunk: [0] dt, [1] cum, [2] gamma, [3] w, [4] e^{cum},
// [5] e^{cum_end - cum} * w, [6] lam
template <typename T>
__global__ void __launch_bounds__(kSimtThreads) scan_simt_kernel(const ScanParams p) {
    extern __shared__ float4 smem4[];
    float* sm = reinterpret_cast<float*>(smem4);
    const int64_t N = p.N, P = p.P, R = p.R, Q = p.Q, L = p.L, half = N / 2;
    const SimtLayout lay = simt_layout(N, P, Q, R);
    float* Hs = sm + lay.H;
    float* Bb = sm + lay.Bb;
    float* Cb = sm + lay.Cb;
    float* Xs = sm + lay.X;
    float* Ss = sm + lay.S;
    float* phir = sm + lay.phi;
    float* rsB = sm + lay.rsB;
    float* rsC = sm + lay.rsC;
    float* sc = sm + lay.sc;

    const int64_t u = blockIdx.x;
    const int64_t bb = u / p.H, hh = u % p.H, g = hh / (p.H / p.G);
    const int tid = threadIdx.x, nth = blockDim.x;
    const int warp = tid >> 5, lane = tid & 31, nwarps = nth >> 5;
    const T* xg = static_cast<const T*>(p.x);
    const T* Bg = static_cast<const T*>(p.B);
    const T* Cg = static_cast<const T*>(p.C);
    const T* thg = static_cast<const T*>(p.theta);
    const float* biasB = p.Bbias ? p.Bbias + hh * R * N : nullptr;
    const float* biasC = p.Cbias ? p.Cbias + hh * R * N : nullptr;
    auto sidx = [&](int64_t t) { return (bb * L + t) * p.H + hh; };  // dt/A/lam index
    const float dtb = p.dt_bias ? p.dt_bias[hh] : 0.f;
    auto dt_at = [&](int64_t t) { return step_dt(p.dt[sidx(t)], dtb, p.flags); };
    auto lam_at = [&](int64_t t) { return step_lam(p.lam[sidx(t)], p.flags); };

    // ---- initial state ----
    for (int64_t e = tid; e < N * P; e += nth) Hs[e] = p.h0 ? p.h0[u * N * P + e] : 0.f;
    for (int64_t i = tid; i < half; i += nth) phir[i] = p.phi0 ? p.phi0[u * half + i] : 0.f;
    __syncthreads();
    if (p.h0 && L > 0) {
        // Fold the stored previous token into the primed state: H += (1-lam_0) dt_0 Bbar_{-1} x_{-1}^T.
        const T* Bp = static_cast<const T*>(p.prevB0) + u * R * N;
        const T* xp = static_cast<const T*>(p.prevx0) + u * R * P;
        for (int64_t e = tid; e < R * N; e += nth) Bb[e] = to_f(Bp[e]);
        for (int64_t e = tid; e < R * P; e += nth) Xs[e] = to_f(xp[e]);
        __syncthreads();
        for (int64_t r = warp; r < R; r += nwarps) {
            float ss = 0.f;
            for (int64_t n = lane; n < N; n += 32) ss += Bb[r * N + n] * Bb[r * N + n];
            ss = warp_sum(ss);
            if (lane == 0) rsB[r] = p.bc_norm ? rsqrtf(ss / static_cast<float>(N) + p.eps) : 1.f;
        }
        __syncthreads();
        for (int64_t i = tid; i < half; i += nth) {
            float s, c;
            sincosf(phir[i], &s, &c);
            for (int64_t r = 0; r < R; ++r) {
                const float u0 = Bb[r * N + i] * rsB[r] + (biasB ? biasB[r * N + i] : 0.f);
                const float u1 = Bb[r * N + i + half] * rsB[r] + (biasB ? biasB[r * N + i + half] : 0.f);
                Bb[r * N + i] = u0 * c + u1 * s;
                Bb[r * N + i + half] = u1 * c - u0 * s;
            }
        }
        __syncthreads();
        const float f = (p.flags & 4u) ? 0.f : (1.f - lam_at(0)) * dt_at(0);
        for (int64_t e = tid; e < N * P; e += nth) {
            const int64_t n = e / P, pp = e % P;
            float acc = 0.f;
            for (int64_t r = 0; r < R; ++r) acc += Bb[r * N + n] * Xs[r * P + pp];
            Hs[e] += f * acc;
        }
        __syncthreads();
    }

    for (int64_t c0 = 0; c0 < L; c0 += Q) {
        const int64_t T_ = (L - c0 < Q) ? (L - c0) : Q;
        const int64_t TR = T_ * R;
        // ---- chunk scalars (one warp; sequential cumsum is cheap at Q <= 128) ----
        if (tid == 0) {
            float cum = 0.f;
            for (int64_t t = 0; t < T_; ++t) {
                const int64_t si = sidx(c0 + t);
                const float d = dt_at(c0 + t), a = p.A[si], l = lam_at(c0 + t);
                cum += d * a;
                const bool zoh = p.flags & 4u;   // zero-order hold: no previous-token term
                const float g = zoh ? zoh_gamma(d, a) : l * d;
                float w = g;
                if (!zoh && c0 + t + 1 < L) w += (1.f - lam_at(c0 + t + 1)) * dt_at(c0 + t + 1);
                sc[8 * t + 0] = d;
                sc[8 * t + 1] = cum;
                sc[8 * t + 2] = g;
                sc[8 * t + 3] = w;
                sc[8 * t + 4] = expf(cum);
            }
            for (int64_t t = 0; t < T_; ++t)
                sc[8 * t + 5] = expf(cum - sc[8 * t + 1]) * sc[8 * t + 3];
        }
        // ---- raw B, C, X of the chunk ----
        for (int64_t e = tid; e < TR * N; e += nth) {
            const int64_t row = e / N, n = e % N, t = row / R, r = row % R;
            const int64_t gi = (((bb * L + c0 + t) * p.G + g) * R + r) * N + n;
            Bb[e] = to_f(Bg[gi]);
            Cb[e] = to_f(Cg[gi]);
        }
        for (int64_t e = tid; e < TR * P; e += nth) {
            const int64_t row = e / P, pp = e % P, t = row / R, r = row % R;
            Xs[e] = to_f(xg[(((bb * L + c0 + t) * p.H + hh) * R + r) * P + pp]);
        }
        __syncthreads();
        // ---- RMS norm scales, one warp per row ----
        for (int64_t row = warp; row < 2 * TR; row += nwarps) {
            const float* src = row < TR ? Bb + row * N : Cb + (row - TR) * N;
            float ss = 0.f;
            for (int64_t n = lane; n < N; n += 32) ss += src[n] * src[n];
            ss = warp_sum(ss);
            if (lane == 0) {
                const float s = p.bc_norm ? rsqrtf(ss / static_cast<float>(N) + p.eps) : 1.f;
                if (row < TR) rsB[row] = s; else rsC[row - TR] = s;
            }
        }
        __syncthreads();
        // ---- cumulative angle and rotation, one thread per pair ----
        for (int64_t i = tid; i < half; i += nth) {
            float ph = phir[i];
            for (int64_t t = 0; t < T_; ++t) {
                const float th = to_f(thg[((bb * L + c0 + t) * p.H + hh) * half + i]);
                ph += sc[8 * t + 0] * th;
                float s, c;
                sincosf(ph, &s, &c);
                for (int64_t r = 0; r < R; ++r) {
                    const int64_t row = t * R + r;
                    float* vb = Bb + row * N;
                    float u0 = vb[i] * rsB[row] + (biasB ? biasB[r * N + i] : 0.f);
                    float u1 = vb[i + half] * rsB[row] + (biasB ? biasB[r * N + i + half] : 0.f);
                    vb[i] = u0 * c + u1 * s;
                    vb[i + half] = u1 * c - u0 * s;
                    float* vc = Cb + row * N;
                    u0 = vc[i] * rsC[row] + (biasC ? biasC[r * N + i] : 0.f);
                    u1 = vc[i + half] * rsC[row] + (biasC ? biasC[r * N + i + half] : 0.f);
                    vc[i] = u0 * c + u1 * s;
                    vc[i + half] = u1 * c - u0 * s;
                }
            }
            phir[i] = ph;
        }
        __syncthreads();
        // ---- masked scores S = (Cbar Bbar^T) o M ----
        for (int64_t e = tid; e < TR * TR; e += nth) {
            const int64_t tr = e / TR, sr = e % TR, t = tr / R, s = sr / R;
            float v = 0.f;
            if (s <= t) {
                const float* cr = Cb + tr * N;
                const float* br = Bb + sr * N;
                float acc = 0.f;
                for (int64_t n = 0; n < N; ++n) acc = fmaf(cr[n], br[n], acc);
                const float m = (s < t) ? expf(sc[8 * t + 1] - sc[8 * s + 1]) * sc[8 * s + 3]
                                        : sc[8 * t + 2];
                v = acc * m;
            }
            Ss[e] = v;
        }
        __syncthreads();
        // ---- outputs: Y = S X + e^{cum} Cbar H0 ----
        T* yg = static_cast<T*>(p.y);
        for (int64_t e = tid; e < TR * P; e += nth) {
            const int64_t tr = e / P, pp = e % P, t = tr / R, r = tr % R;
            float acc = 0.f;
            const int64_t smax = (t + 1) * R;
            for (int64_t sr = 0; sr < smax; ++sr) acc = fmaf(Ss[tr * TR + sr], Xs[sr * P + pp], acc);
            float off = 0.f;
            const float* cr = Cb + tr * N;
            for (int64_t n = 0; n < N; ++n) off = fmaf(cr[n], Hs[n * P + pp], off);
            acc = fmaf(sc[8 * t + 4], off, acc);
            yg[(((bb * L + c0 + t) * p.H + hh) * R + r) * P + pp] = from_f<T>(acc);
        }
        __syncthreads();
        // ---- chunk-end state: H1 = e^{cum_end} H0 + Bbar^T diag(e^{cum_end-cum} w) X ----
        const float eend = sc[8 * (T_ - 1) + 4];
        for (int64_t e = tid; e < N * P; e += nth) {
            const int64_t n = e / P, pp = e % P;
            float acc = 0.f;
            for (int64_t sr = 0; sr < TR; ++sr)
                acc = fmaf(Bb[sr * N + n] * sc[8 * (sr / R) + 5], Xs[sr * P + pp], acc);
            Hs[e] = fmaf(eend, Hs[e], acc);
        }
        __syncthreads();
    }

    // ---- final state ----
    if (p.h1)
        for (int64_t e = tid; e < N * P; e += nth) p.h1[u * N * P + e] = Hs[e];
    if (p.phi1)
        for (int64_t i = tid; i < half; i += nth) p.phi1[u * half + i] = phir[i];
    if (L > 0) {
        if (p.prevB1) {
            T* dst = static_cast<T*>(p.prevB1) + u * R * N;
            const T* src = Bg + ((bb * L + L - 1) * p.G + g) * R * N;
            for (int64_t e = tid; e < R * N; e += nth) dst[e] = src[e];
        }
        if (p.prevx1) {
            T* dst = static_cast<T*>(p.prevx1) + u * R * P;
            const T* src = xg + ((bb * L + L - 1) * p.H + hh) * R * P;
            for (int64_t e = tid; e < R * P; e += nth) dst[e] = src[e];
        }
    }
}

}  // namespace

size_t simt_scan_smem_bytes(const ScanParams& p) {
    return sizeof(float) * static_cast<size_t>(simt_layout(p.N, p.P, p.Q, p.R).total);
}

cudaError_t launch_scan_simt(const ScanParams& p, bool bf16, cudaStream_t s) {
    if (p.b * p.H == 0) return cudaSuccess;
    const size_t smem = simt_scan_smem_bytes(p);
    auto k = bf16 ? scan_simt_kernel<__nv_bfloat16> : scan_simt_kernel<float>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    k<<<static_cast<unsigned>(p.b * p.H), kSimtThreads, smem, s>>>(p);
    return cudaGetLastError();
}

}  // namespace m3
