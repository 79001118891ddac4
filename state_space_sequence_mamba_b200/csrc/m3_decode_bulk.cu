// One-token decode step, persistent form with bulk asynchronous copies.
//
// Same arithmetic as m3_decode.cu (one iteration of the exponential-trapezoidal, rotated-frame
// recurrence per (batch, head) unit: "Mamba-3: Improved Sequence Modeling using State Space
// Principles", Sec. 3.1.1 Prop. 1, Sec. 3.2.2 Prop. 4, Appendix C), organised for HBM
// bandwidth: each CTA walks a strided list of units. While it updates one unit, the bulk-copy
// (TMA) engine already brings the next unit's fp32 state and all of its small inputs into the
// other half of a shared-memory double buffer, and sends the previous unit's updated state
// back. The big state stream therefore never waits on registers or on the prologue
// (norms, angles, rotations) of the unit being computed.
//
// Used for bf16 inputs whose per-unit state fits the 32 KB buffer (N * P <= 8192).
#include "m3_common.cuh"
#include "m3_internal.h"
#include "m3_sm100.cuh"

namespace m3 {
namespace {

using namespace sm100;

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

__host__ __device__ inline uint32_t rup(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

// Byte layout of one buffer half (every piece 16-byte aligned for bulk copies).
struct BufLayout {
    uint32_t h, x, xp, bp, b, c, th, phi, total;
};
__host__ __device__ inline BufLayout buf_layout(int N, int P, int R) {
    BufLayout l;
    uint32_t o = 0;
    l.h = o; o += N * P * 4;
    l.x = o; o += rup(R * P * 2, 16);
    l.xp = o; o += rup(R * P * 2, 16);
    l.bp = o; o += rup(R * N * 2, 16);
    l.b = o; o += rup(R * N * 2, 16);
    l.c = o; o += rup(R * N * 2, 16);
    l.th = o; o += rup(N, 16);           // N/2 bf16
    l.phi = o; o += rup(N * 2, 16);      // N/2 fp32
    l.total = rup(o, 128);
    return l;
}
// Shared scratch after the two buffers (floats).
struct ScratchLayout {
    uint32_t vb, vbp, cc, rs, ypart, phin, sc, total;  // float offsets
};
__host__ __device__ inline ScratchLayout scratch_layout(int N, int P, int R) {
    ScratchLayout l;
    uint32_t o = 0;
    l.vb = o; o += R * N;
    l.vbp = o; o += R * N;
    l.cc = o; o += R * N;
    l.rs = o; o += 4 * R;
    l.ypart = o; o += kWarps * R * P;
    l.phin = o; o += N / 2;
    l.sc = o; o += 8;                    // two slots of (dt, A, lam, pad)
    l.total = o;
    return l;
}

// x reduced by a whole number of turns into [-pi, pi]: Cody-Waite reduction with 2*pi split
// into an exactly representable head and a tail (Cody & Waite, "Software Manual for the
// Elementary Functions", 1980); the hardware sine/cosine then sees a small argument.
__device__ __forceinline__ float reduce_turns(float x) {
    const float k = rintf(x * 0.15915494309189535f);
    return fmaf(-k, 1.9353071795864769e-3f, fmaf(-k, 6.28125f, x));
}

__device__ __forceinline__ void bulk_store(void* gdst, const void* ssrc, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                 :: "l"(gdst), "r"(smem_u32(ssrc)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bulk_commit() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read_all() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// kRaw: dt and lam arrive raw (m3_dims.flags); the step scalars apply softplus / sigmoid.
template <int R, bool kRaw>
__global__ void __launch_bounds__(kThreads, 2)
decode_bulk_kernel(const ScanParams p, const int n_units) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~static_cast<uintptr_t>(127));
    const int N = static_cast<int>(p.N), P = static_cast<int>(p.P), half = N / 2;
    const BufLayout bl = buf_layout(N, P, R);
    const ScratchLayout sl = scratch_layout(N, P, R);
    float* scr = reinterpret_cast<float*>(sm + 2 * bl.total);
    float* vB = scr + sl.vb;
    float* vBp = scr + sl.vbp;
    float* cC = scr + sl.cc;
    float* rs = scr + sl.rs;
    float* ypart = scr + sl.ypart;
    float* phin = scr + sl.phin;
    float* sc = scr + sl.sc;
    __shared__ uint64_t bar[2];
    __shared__ int s_abort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int PV = P / 4, RP = kThreads / PV;
    const int pc = tid % PV, r0 = tid / PV;
    const __nv_bfloat16* xg = static_cast<const __nv_bfloat16*>(p.x);
    const __nv_bfloat16* Bg = static_cast<const __nv_bfloat16*>(p.B);
    const __nv_bfloat16* Cg = static_cast<const __nv_bfloat16*>(p.C);
    const __nv_bfloat16* thg = static_cast<const __nv_bfloat16*>(p.theta);
    const __nv_bfloat16* pBg = static_cast<const __nv_bfloat16*>(p.prevB0);
    const __nv_bfloat16* pxg = static_cast<const __nv_bfloat16*>(p.prevx0);
    const uint32_t tx = static_cast<uint32_t>(N * P * 4 + 2 * R * P * 2 + 3 * R * N * 2 + half * 2 +
                                              half * 4);

    auto issue = [&](int u, int b) {  // every per-unit input of unit u into buffer half b
        uint8_t* base = sm + b * bl.total;
        const int64_t bb = u / p.H, hh = u % p.H, g = hh / (p.H / p.G);
        mbar_arrive_expect_tx(&bar[b], tx);
        bulk_load(base + bl.h, p.h0 + static_cast<int64_t>(u) * N * P, N * P * 4, &bar[b]);
        bulk_load(base + bl.x, xg + static_cast<int64_t>(u) * R * P, R * P * 2, &bar[b]);
        bulk_load(base + bl.xp, pxg + static_cast<int64_t>(u) * R * P, R * P * 2, &bar[b]);
        bulk_load(base + bl.bp, pBg + static_cast<int64_t>(u) * R * N, R * N * 2, &bar[b]);
        bulk_load(base + bl.b, Bg + (bb * p.G + g) * R * N, R * N * 2, &bar[b]);
        bulk_load(base + bl.c, Cg + (bb * p.G + g) * R * N, R * N * 2, &bar[b]);
        bulk_load(base + bl.th, thg + static_cast<int64_t>(u) * half, half * 2, &bar[b]);
        bulk_load(base + bl.phi, p.phi0 + static_cast<int64_t>(u) * half, half * 4, &bar[b]);
    };

    int u = blockIdx.x;
    // thread 0: loads issued into each buffer half, and how many of them were waited for
    int issued[2] = {0, 0}, waited[2] = {0, 0};
    if (tid == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        fence_mbar_init();
        s_abort = 0;
        if (u < n_units) {
            issue(u, 0);
            issued[0] = 1;
            sc[0] = step_dt<kRaw>(p.dt[u], (kRaw && p.dt_bias) ? p.dt_bias[u % static_cast<int>(p.H)] : 0.f,
                                    p.flags);
            sc[1] = p.A[u];
            sc[2] = step_lam<kRaw>(p.lam[u], p.flags);
        }
    }
    __syncthreads();

    for (int i = 0; u < n_units; ++i, u += gridDim.x) {
        const int b = i & 1;
        uint8_t* base = sm + b * bl.total;
        const int un = u + gridDim.x;
        float snext[4] = {0.f, 0.f, 0.f, 0.f};   // raw dt, A, raw lam, dt bias
        if (tid == 0) {
            // the other half held the previous unit, whose state is being stored from it
            // ...and is free for the next unit once that store has read it: request the next
            // unit before waiting for this one, so two units stream in at once
            bulk_wait_read_all();
            if (un < n_units) {
                issue(un, b ^ 1);
                ++issued[b ^ 1];
                snext[0] = p.dt[un];
                snext[1] = p.A[un];
                snext[2] = p.lam[un];
                if constexpr (kRaw) snext[3] = p.dt_bias ? p.dt_bias[un % static_cast<int>(p.H)] : 0.f;
            }
            if (mbar_wait_sleep(&bar[b], (i >> 1) & 1)) ++waited[b];
            else s_abort = 1;
        }
        __syncthreads();
        if (s_abort) break;
        (void)mbar_try_wait(smem_u32(&bar[b]), (i >> 1) & 1);  // completed: orders the data

        const __nv_bfloat16* sB = reinterpret_cast<const __nv_bfloat16*>(base + bl.b);
        const __nv_bfloat16* sC = reinterpret_cast<const __nv_bfloat16*>(base + bl.c);
        const __nv_bfloat16* sBp = reinterpret_cast<const __nv_bfloat16*>(base + bl.bp);
        const float d = sc[4 * b + 0], a = sc[4 * b + 1], lm = sc[4 * b + 2];
        const float al = expf(d * a);
        float be = (1.f - lm) * d * al, ga = lm * d;
        if constexpr (kRaw) {
            if (p.flags & 4u) {   // zero-order hold: no previous-token term
                be = 0.f;
                ga = zoh_gamma(d, a);
            }
        }

        // ---- RMS scales of B, C and the stored previous B, one warp per vector ----
        if (p.bc_norm) {
            for (int v = warp; v < 3 * R; v += kWarps) {
                const __nv_bfloat16* src = (v < R) ? sB + v * N : (v < 2 * R) ? sC + (v - R) * N
                                                                             : sBp + (v - 2 * R) * N;
                float ss = 0.f;
                for (int n = 2 * lane; n < N; n += 64) {
                    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(src + n));
                    ss = fmaf(f.x, f.x, fmaf(f.y, f.y, ss));
                }
                ss = warp_sum(ss);
                if (lane == 0) rs[v] = rsqrtf(ss / static_cast<float>(N) + p.eps);
            }
        } else if (tid < 3 * R) {
            rs[tid] = 1.f;
        }
        __syncthreads();
        // ---- angles and rotations, pair i = (i, i + N/2); vectors stored [n][R] ----
        {
            const int64_t hh = u % p.H;
            const float* bB = p.Bbias ? p.Bbias + hh * R * N : nullptr;
            const float* bC = p.Cbias ? p.Cbias + hh * R * N : nullptr;
            const __nv_bfloat16* sth = reinterpret_cast<const __nv_bfloat16*>(base + bl.th);
            const float* sphi = reinterpret_cast<const float*>(base + bl.phi);
            // items (k, r): k in [0, half) rotates B and C of rank r by the new angle, k in
            // [half, 2 half) the stored previous B by the old one
            for (int it = tid; it < 2 * half * R; it += kThreads) {
                const int k = it / R, r = it - k * R;
                const bool cur = k < half;
                const int i = cur ? k : k - half;
                const float ph_old = sphi[i];
                const float ph = cur ? ph_old + d * __bfloat162float(sth[i]) : ph_old;
                float sn, cn;
                __sincosf(reduce_turns(ph), &sn, &cn);
                const int a0 = r * N + i, a1 = a0 + half;
                const int o0 = i * R + r, o1 = (i + half) * R + r;
                if (cur) {
                    float u0 = fmaf(__bfloat162float(sB[a0]), rs[r], bB ? bB[a0] : 0.f);
                    float u1 = fmaf(__bfloat162float(sB[a1]), rs[r], bB ? bB[a1] : 0.f);
                    vB[o0] = ga * (u0 * cn + u1 * sn);
                    vB[o1] = ga * (u1 * cn - u0 * sn);
                    u0 = fmaf(__bfloat162float(sC[a0]), rs[R + r], bC ? bC[a0] : 0.f);
                    u1 = fmaf(__bfloat162float(sC[a1]), rs[R + r], bC ? bC[a1] : 0.f);
                    cC[o0] = u0 * cn + u1 * sn;
                    cC[o1] = u1 * cn - u0 * sn;
                    if (r == 0) phin[i] = ph;
                } else {
                    const float u0 = fmaf(__bfloat162float(sBp[a0]), rs[2 * R + r], bB ? bB[a0] : 0.f);
                    const float u1 = fmaf(__bfloat162float(sBp[a1]), rs[2 * R + r], bB ? bB[a1] : 0.f);
                    vBp[o0] = be * (u0 * cn + u1 * sn);
                    vBp[o1] = be * (u1 * cn - u0 * sn);
                }
            }
        }
        __syncthreads();

        // ---- state update in place and readout ----
        float2 y01[R], y23[R];
#pragma unroll
        for (int r = 0; r < R; ++r) y01[r] = y23[r] = make_float2(0.f, 0.f);
        {
            const __nv_bfloat16* sx = reinterpret_cast<const __nv_bfloat16*>(base + bl.x);
            const __nv_bfloat16* sxp = reinterpret_cast<const __nv_bfloat16*>(base + bl.xp);
            float4 xv[R], xpv[R];
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const int o = r * P + 4 * pc;
                xv[r] = make_float4(__bfloat162float(sx[o]), __bfloat162float(sx[o + 1]),
                                    __bfloat162float(sx[o + 2]), __bfloat162float(sx[o + 3]));
                xpv[r] = make_float4(__bfloat162float(sxp[o]), __bfloat162float(sxp[o + 1]),
                                     __bfloat162float(sxp[o + 2]), __bfloat162float(sxp[o + 3]));
            }
            float4* hs = reinterpret_cast<float4*>(base + bl.h);
            auto row_vals = [&](const float* v, int n, float (&o)[R]) {
                if constexpr (R % 4 == 0) {
#pragma unroll
                    for (int r = 0; r < R; r += 4) {
                        const float4 q = *reinterpret_cast<const float4*>(v + n * R + r);
                        o[r] = q.x; o[r + 1] = q.y; o[r + 2] = q.z; o[r + 3] = q.w;
                    }
                } else if constexpr (R == 2) {
                    const float2 q = *reinterpret_cast<const float2*>(v + n * R);
                    o[0] = q.x; o[1] = q.y;
                } else {
                    o[0] = v[n];
                }
            };
            // packed fp32 pairs (fma.rn.f32x2): columns (4 pc, 4 pc + 1) and (4 pc + 2, 4 pc + 3)
            float2 x01[R], x23[R], xp01[R], xp23[R];
#pragma unroll
            for (int r = 0; r < R; ++r) {
                x01[r] = make_float2(xv[r].x, xv[r].y);
                x23[r] = make_float2(xv[r].z, xv[r].w);
                xp01[r] = make_float2(xpv[r].x, xpv[r].y);
                xp23[r] = make_float2(xpv[r].z, xpv[r].w);
            }
            const float2 al2 = make_float2(al, al);
            auto update = [&](int n) {
                float a2[R], c2[R], cc[R];
                row_vals(vBp, n, a2);
                row_vals(vB, n, c2);
                row_vals(cC, n, cc);
                const float4 h = hs[n * PV + pc];
                float2 h01 = __fmul2_rn(make_float2(h.x, h.y), al2);
                float2 h23 = __fmul2_rn(make_float2(h.z, h.w), al2);
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const float2 cr = make_float2(c2[r], c2[r]), ar = make_float2(a2[r], a2[r]);
                    h01 = __ffma2_rn(ar, xp01[r], __ffma2_rn(cr, x01[r], h01));
                    h23 = __ffma2_rn(ar, xp23[r], __ffma2_rn(cr, x23[r], h23));
                }
                hs[n * PV + pc] = make_float4(h01.x, h01.y, h23.x, h23.y);
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const float2 c = make_float2(cc[r], cc[r]);
                    y01[r] = __ffma2_rn(h01, c, y01[r]);
                    y23[r] = __ffma2_rn(h23, c, y23[r]);
                }
            };
            int n = r0;
            for (; n + RP < N; n += 2 * RP) {
                update(n);
                update(n + RP);
            }
            for (; n < N; n += RP) update(n);
        }
        fence_proxy_async();  // the updated state is read by the bulk store

        float yacc[R][4];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            yacc[r][0] = y01[r].x; yacc[r][1] = y01[r].y; yacc[r][2] = y23[r].x; yacc[r][3] = y23[r].y;
        }
        // partial outputs: lanes sharing a column group differ in the bits above log2(PV)
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
        if (tid == 0) {
            bulk_store(p.h1 + static_cast<int64_t>(u) * N * P, base + bl.h, N * P * 4);
            bulk_commit();
        }
        {
            __nv_bfloat16* yout = static_cast<__nv_bfloat16*>(p.y) + static_cast<int64_t>(u) * R * P;
            for (int e = tid; e < R * P; e += kThreads) {
                const int r = e / P, col = e % P;
                float acc = 0.f;
                for (int w = 0; w < kWarps; ++w) acc += ypart[(w * R + r) * P + col];
                yout[e] = __float2bfloat16_rn(acc);
            }
            for (int k = tid; k < half; k += kThreads) p.phi1[static_cast<int64_t>(u) * half + k] = phin[k];
            const __nv_bfloat16* sx = reinterpret_cast<const __nv_bfloat16*>(base + bl.x);
            __nv_bfloat16* pb1 = static_cast<__nv_bfloat16*>(p.prevB1) + static_cast<int64_t>(u) * R * N;
            __nv_bfloat16* px1 = static_cast<__nv_bfloat16*>(p.prevx1) + static_cast<int64_t>(u) * R * P;
            for (int e = tid; e < R * N / 8; e += kThreads)
                reinterpret_cast<uint4*>(pb1)[e] = reinterpret_cast<const uint4*>(sB)[e];
            for (int e = tid; e < R * P / 8; e += kThreads)
                reinterpret_cast<uint4*>(px1)[e] = reinterpret_cast<const uint4*>(sx)[e];
        }
        if (tid == 0) {
            sc[4 * (b ^ 1) + 0] = step_dt<kRaw>(snext[0], snext[3], p.flags);
            sc[4 * (b ^ 1) + 1] = snext[1];
            sc[4 * (b ^ 1) + 2] = step_lam<kRaw>(snext[2], p.flags);
        }
        __syncthreads();
    }
    if (tid == 0) {
        if (s_abort && p.status) atomicExch(p.status, 1);
        bulk_wait_all();
        // inputs requested but never waited for (only after a wait gave up): let them land
        for (int h = 0; h < 2; ++h)
            for (int k = waited[h]; k < issued[h]; ++k)
                (void)mbar_wait(&bar[h], static_cast<uint32_t>(k & 1), 200000000LL);
    }
    __syncthreads();
}

}  // namespace

bool decode_bulk_supported(const ScanParams& p, bool bf16) {
    return bf16 && p.N * p.P <= 8192 && (p.R == 1 || p.R == 2 || p.R == 4 || p.R == 8);
}

size_t decode_bulk_smem_bytes(const ScanParams& p) {
    const int N = static_cast<int>(p.N), P = static_cast<int>(p.P), R = static_cast<int>(p.R);
    return 2 * buf_layout(N, P, R).total + 4 * scratch_layout(N, P, R).total + 128;
}

template <int R>
static cudaError_t launch_bulk_t(const ScanParams& p, cudaStream_t s) {
    const int sms = device_sm_count();
    const size_t smem = decode_bulk_smem_bytes(p);
    auto k = p.flags ? decode_bulk_kernel<R, true> : decode_bulk_kernel<R, false>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const int units = static_cast<int>(p.b * p.H);
    const int grid = units < 2 * sms ? units : 2 * sms;
    k<<<grid, kThreads, smem, s>>>(p, units);
    return cudaGetLastError();
}

cudaError_t launch_decode_bulk(const ScanParams& p, cudaStream_t s) {
    switch (p.R) {
        case 1: return launch_bulk_t<1>(p, s);
        case 2: return launch_bulk_t<2>(p, s);
        case 4: return launch_bulk_t<4>(p, s);
        case 8: return launch_bulk_t<8>(p, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace m3
