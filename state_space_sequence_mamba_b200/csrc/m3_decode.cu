// One-token decode step of the Mamba-3 SSM core.
//
// Per (batch, head) unit this is one iteration of the exponential-trapezoidal recurrence in
// the rotated frame ("Mamba-3: Improved Sequence Modeling using State Space Principles",
// Sec. 3.1.1 Prop. 1, Sec. 3.2.2 Prop. 4, Appendix C for the rank-R state update):
//     Phi'  = Phi + dt theta
//     h     = alpha h + beta sum_r Bbar_prev[r] x_prev[r]^T + gamma sum_r Bbar[r] x[r]^T
//     y[r]  = h^T Cbar[r]
// with Bbar = R(Phi')^T (norm(B) + bias_B), Cbar likewise and Bbar_prev = R(Phi)^T applied to
// the previous token's normalised, biased B.
//
// The step is bound by HBM: each unit streams its fp32 N x P state in and out once (32 KB
// each way at N = 128, P = 64), everything else is < 1.5 % of the bytes. One CTA owns one
// unit. The state is read with 128-bit loads in the order it is stored (rows of P floats), the
// first rows are requested before the prologue (norms, angles, rotations) runs so that the
// loads are in flight while it computes, and the rank-2R update plus the readout are plain
// FP32 FMAs on registers (for R = 4: ~13 FMA per state element, well under the time the
// bytes take).
#include "m3_common.cuh"
#include "m3_internal.h"

namespace m3 {

namespace {

constexpr int kDecodeThreads = 256;
constexpr int kRowsInFlight = 8;  // state rows (float4 each) a thread keeps in flight

template <int R, typename T>
__global__ void __launch_bounds__(kDecodeThreads)
decode_kernel(const ScanParams p, const int rows_per_pass) {
    extern __shared__ float4 smem4[];
    float* sm = reinterpret_cast<float*>(smem4);
    const int N = static_cast<int>(p.N), P = static_cast<int>(p.P), half = N / 2;
    const int64_t u = blockIdx.x;
    const int64_t bb = u / p.H, hh = u % p.H, g = hh / (p.H / p.G);
    const int tid = threadIdx.x;
    const int PV = P / 4;             // float4 column groups per state row (4..32)
    const int RP = rows_per_pass;      // rows covered by the block in one pass
    const bool active = true;          // PV * RP == blockDim.x for the supported P
    const int pc = tid % PV, r0 = tid / PV;

    // ---- issue the first state loads before anything else ----
    const float4* hin = reinterpret_cast<const float4*>(p.h0 + u * N * P);
    float4* hout = reinterpret_cast<float4*>(p.h1 + u * N * P);
    float4 hv[kRowsInFlight];
    if (active) {
#pragma unroll
        for (int k = 0; k < kRowsInFlight; ++k) {
            const int n = r0 + k * RP;
            if (n < N) hv[k] = __ldcs(hin + n * PV + pc);
        }
    }

    // ---- shared memory carve-up ----
    float* vB = sm;              // [R][N]  gamma * Bbar
    float* vBp = vB + R * N;     // [R][N]  beta * Bbar_prev
    float* cC = vBp + R * N;     // [R][N]  Cbar
    float* rawB = cC + R * N;    // [R][N]
    float* rawC = rawB + R * N;  // [R][N]
    float* rawBp = rawC + R * N; // [R][N]
    float* xs = rawBp + R * N;   // [R][P]
    float* xps = xs + R * P;     // [R][P]
    float* rs = xps + R * P;     // [3R]  norm scales of B, C, B_prev
    float* scal = rs + 3 * R;    // alpha, beta, gamma, dt
    float* ypart = scal + 4;     // [warps][R][P]

    const T* Bin = static_cast<const T*>(p.B) + (bb * p.G + g) * R * N;
    const T* Cin = static_cast<const T*>(p.C) + (bb * p.G + g) * R * N;
    const T* Bpin = static_cast<const T*>(p.prevB0) + u * R * N;
    const T* xin = static_cast<const T*>(p.x) + u * R * P;
    const T* xpin = static_cast<const T*>(p.prevx0) + u * R * P;
    for (int i = tid; i < R * N; i += blockDim.x) {
        rawB[i] = to_f(Bin[i]);
        rawC[i] = to_f(Cin[i]);
        rawBp[i] = to_f(Bpin[i]);
    }
    for (int i = tid; i < R * P; i += blockDim.x) {
        if (p.proj) {   // X[r][p] = W_X[h][r][p] X'[p] (Appendix C)
            const int pp = i % P;
            xs[i] = p.WX[hh * R * P + i] * to_f(static_cast<const T*>(p.xprj)[u * P + pp]);
        } else {
            xs[i] = to_f(xin[i]);
        }
        xps[i] = to_f(xpin[i]);
    }
    if (tid == 0) {
        const float d = step_dt(p.dt[u], p.dt_bias ? p.dt_bias[u % p.H] : 0.f, p.flags);
        const float a = p.A[u], l = step_lam(p.lam[u], p.flags);
        const float al = expf(d * a);
        scal[0] = al;
        const bool zoh = p.flags & 4u;   // zero-order hold: no previous-token term
        scal[1] = zoh ? 0.f : (1.f - l) * d * al;
        scal[2] = zoh ? zoh_gamma(d, a) : l * d;
        scal[3] = d;
    }
    __syncthreads();

    // ---- RMS norm scales, one warp per vector ----
    const int warp = tid >> 5, lane = tid & 31, nwarps = blockDim.x >> 5;
    for (int v = warp; v < 3 * R; v += nwarps) {
        const float* src = (v < R) ? rawB + v * N : (v < 2 * R) ? rawC + (v - R) * N
                                                                  : rawBp + (v - 2 * R) * N;
        float ss = 0.f;
        for (int i = lane; i < N; i += 32) ss += src[i] * src[i];
        ss = warp_sum(ss);
        if (lane == 0) rs[v] = p.bc_norm ? rsqrtf(ss / static_cast<float>(N) + p.eps) : 1.f;
    }
    __syncthreads();

    // ---- angles and rotations (pair i = (i, i + N/2)) ----
    {
        const float al = scal[0], be = scal[1], ga = scal[2], d = scal[3];
        (void)al;
        const float* bB = p.Bbias ? p.Bbias + hh * R * N : nullptr;
        const float* bC = p.Cbias ? p.Cbias + hh * R * N : nullptr;
        const T* th = static_cast<const T*>(p.theta) + u * half;
        for (int i = tid; i < half; i += blockDim.x) {
            const float ph_old = p.phi0[u * half + i];
            const float ph_new = ph_old + d * to_f(th[i]);
            float sn, cn, so, co;
            sincosf(ph_new, &sn, &cn);
            sincosf(ph_old, &so, &co);
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const int a0 = r * N + i, a1 = a0 + half;
                float u0 = rawB[a0] * rs[r] + (bB ? bB[a0] : 0.f);
                float u1 = rawB[a1] * rs[r] + (bB ? bB[a1] : 0.f);
                vB[a0] = ga * (u0 * cn + u1 * sn);
                vB[a1] = ga * (u1 * cn - u0 * sn);
                u0 = rawC[a0] * rs[R + r] + (bC ? bC[a0] : 0.f);
                u1 = rawC[a1] * rs[R + r] + (bC ? bC[a1] : 0.f);
                cC[a0] = u0 * cn + u1 * sn;
                cC[a1] = u1 * cn - u0 * sn;
                u0 = rawBp[a0] * rs[2 * R + r] + (bB ? bB[a0] : 0.f);
                u1 = rawBp[a1] * rs[2 * R + r] + (bB ? bB[a1] : 0.f);
                vBp[a0] = be * (u0 * co + u1 * so);
                vBp[a1] = be * (u1 * co - u0 * so);
            }
            if (p.phi1) p.phi1[u * half + i] = ph_new;
        }
    }
    __syncthreads();

    // ---- state update and readout ----
    float yacc[R][4];
#pragma unroll
    for (int r = 0; r < R; ++r) yacc[r][0] = yacc[r][1] = yacc[r][2] = yacc[r][3] = 0.f;
    if (active) {
        const float al = scal[0];
        float4 xv[R], xpv[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            xv[r] = reinterpret_cast<const float4*>(xs + r * P)[pc];
            xpv[r] = reinterpret_cast<const float4*>(xps + r * P)[pc];
        }
        for (int base = 0; base < N; base += kRowsInFlight * RP) {
            if (base > 0) {
#pragma unroll
                for (int k = 0; k < kRowsInFlight; ++k) {
                    const int n = base + r0 + k * RP;
                    if (n < N) hv[k] = __ldcs(hin + n * PV + pc);
                }
            }
#pragma unroll
            for (int k = 0; k < kRowsInFlight; ++k) {
                const int n = base + r0 + k * RP;
                if (n < N) {
                    float4 h = hv[k];
                    h.x *= al; h.y *= al; h.z *= al; h.w *= al;
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        const float a = vBp[r * N + n], c = vB[r * N + n];
                        h.x = fmaf(a, xpv[r].x, fmaf(c, xv[r].x, h.x));
                        h.y = fmaf(a, xpv[r].y, fmaf(c, xv[r].y, h.y));
                        h.z = fmaf(a, xpv[r].z, fmaf(c, xv[r].z, h.z));
                        h.w = fmaf(a, xpv[r].w, fmaf(c, xv[r].w, h.w));
                    }
                    if (p.h1) __stcs(hout + n * PV + pc, h);
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        const float cc = cC[r * N + n];
                        yacc[r][0] = fmaf(h.x, cc, yacc[r][0]);
                        yacc[r][1] = fmaf(h.y, cc, yacc[r][1]);
                        yacc[r][2] = fmaf(h.z, cc, yacc[r][2]);
                        yacc[r][3] = fmaf(h.w, cc, yacc[r][3]);
                    }
                }
            }
        }
    }
    // Reduce partial outputs over the rows. P is a power of two in [16, 128], so PV = P/4
    // divides 32 and every thread is active: lanes sharing a column group differ in the bits
    // above log2(PV). Sum those within the warp, then across warps through shared memory.
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
        if (off < PV) break;
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int j = 0; j < 4; ++j)
                yacc[r][j] += __shfl_xor_sync(0xffffffffu, yacc[r][j], off);
    }
    if (lane < PV) {
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int j = 0; j < 4; ++j) ypart[(warp * R + r) * P + lane * 4 + j] = yacc[r][j];
    }
    __syncthreads();
    if (p.proj) {
        // O'[p] = sum_r W_O[h][r][p] Y[r][p] SiLU(W_Z[h][r][p] Z'[p]) (Appendix C)
        T* oout = static_cast<T*>(p.y) + u * P;
        for (int col = tid; col < P; col += blockDim.x) {
            const float zp = to_f(static_cast<const T*>(p.zprj)[u * P + col]);
            float o = 0.f;
            for (int r = 0; r < R; ++r) {
                float acc = 0.f;
                for (int w = 0; w < nwarps; ++w) acc += ypart[(w * R + r) * P + col];
                const float z = p.WZ[hh * R * P + r * P + col] * zp;
                o = fmaf(p.WO[hh * R * P + r * P + col], acc * z / (1.f + __expf(-z)), o);
            }
            oout[col] = from_f<T>(o);
        }
    } else {
        T* yout = static_cast<T*>(p.y) + u * R * P;
        for (int e = tid; e < R * P; e += blockDim.x) {
            const int r = e / P, col = e % P;
            float acc = 0.f;
            for (int w = 0; w < nwarps; ++w) acc += ypart[(w * R + r) * P + col];
            yout[e] = from_f<T>(acc);
        }
    }
    // ---- previous-token fields of the new state ----
    if (p.prevB1) {
        T* dst = static_cast<T*>(p.prevB1) + u * R * N;
        for (int i = tid; i < R * N; i += blockDim.x) dst[i] = Bin[i];
    }
    if (p.prevx1) {   // with the projections, the expanded X
        T* dst = static_cast<T*>(p.prevx1) + u * R * P;
        for (int i = tid; i < R * P; i += blockDim.x) dst[i] = p.proj ? from_f<T>(xs[i]) : xin[i];
    }
}

int rows_per_pass_for(int P) { return kDecodeThreads / (P / 4); }

}  // namespace

size_t decode_smem_bytes(const ScanParams& p) {
    const int R = static_cast<int>(p.R), N = static_cast<int>(p.N), P = static_cast<int>(p.P);
    const int warps = kDecodeThreads / 32;
    return sizeof(float) * (static_cast<size_t>(6) * R * N + 2 * R * P + 3 * R + 4 +
                            static_cast<size_t>(warps) * R * P);
}

template <int R, typename T>
static cudaError_t launch_decode_t(const ScanParams& p, cudaStream_t s) {
    const size_t smem = decode_smem_bytes(p);
    auto k = decode_kernel<R, T>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return e;
    }
    const int P = static_cast<int>(p.P);
    k<<<static_cast<unsigned>(p.b * p.H), kDecodeThreads, smem, s>>>(p, rows_per_pass_for(P));
    return cudaGetLastError();
}

cudaError_t launch_decode(const ScanParams& p, bool bf16, cudaStream_t s) {
    if (p.b * p.H == 0) return cudaSuccess;
    if (decode_tc_supported(p, bf16)) return launch_decode_tc(p, s);
    if (!p.proj && decode_bulk_supported(p, bf16)) return launch_decode_bulk(p, s);
    switch (p.R) {
        case 1: return bf16 ? launch_decode_t<1, __nv_bfloat16>(p, s) : launch_decode_t<1, float>(p, s);
        case 2: return bf16 ? launch_decode_t<2, __nv_bfloat16>(p, s) : launch_decode_t<2, float>(p, s);
        case 4: return bf16 ? launch_decode_t<4, __nv_bfloat16>(p, s) : launch_decode_t<4, float>(p, s);
        case 8: return bf16 ? launch_decode_t<8, __nv_bfloat16>(p, s) : launch_decode_t<8, float>(p, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace m3
