// Chunked prefill scan on the sm_100a tensor cores (tcgen05.mma, accumulators in TMEM).
//
// Method ("Mamba-3: Improved Sequence Modeling using State Space Principles", Sec. 3.1.3
// eq. 7 for the masked parallel form, Sec. 3.3 for the chunked algorithm and MIMO, Appendix
// B.3 for the rotated frame): the state carried between chunks is the primed state
//     h'_t = h~_t + (1 - lam_{t+1}) dt_{t+1} v_t,   v_t = sum_r Bbar_t[r] x_t[r]^T,
// which obeys h'_t = alpha_t h'_{t-1} + w_t v_t with w_t = gamma_t + (1 - lam_{t+1}) dt_{t+1}
// (w = gamma for the sequence's last token). Per chunk of Q tokens (64 rows = Q x R), from
// H0 = h' before the chunk and cum = chunk-local inclusive sum of dt*A:
//     S   = Cbar Bbar^T                                  (tensor core, M64 N64 K128)
//     Yo  = Cbar H0                                      (tensor core, M64 N64 K128)
//     dH  = Bbar^T (diag(e^{cum_end - cum} w) X)         (tensor core, M128 N64 K64)
//     P   = S o M,  M[t,s] = e^{cum_t-cum_s} w_s (s<t), gamma_t (s=t), 0 (s>t)   (CUDA cores)
//     Yd  = P X                                          (tensor core, M64 N64 K64)
//     y   = Yd + diag(e^{cum}) Yo ;  H1 = e^{cum_end} H0 + dH   (CUDA cores, fp32)
// MIMO rows are (token, rank) pairs, the token mask applied to full R x R blocks.
//
// Data flow per CTA (one (batch, head) unit, 8 warps): X arrives by TMA in the 128-byte
// swizzled layout the MMA reads; B, C, theta are read from global (B and C are shared by all
// heads, so they come from L2), normalised, biased and rotated on the CUDA cores straight into
// swizzled bf16 operand tiles; the fp32 state lives in registers (row n of the state in lane n
// of the TMEM datapath, matching the dH accumulator) and is rounded to bf16 only as the Yo
// operand. All waits are bounded; a timeout sets the status word and the CTA exits cleanly.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "m3_common.cuh"
#include "m3_internal.h"
#include "m3_sm100.cuh"

namespace m3 {

namespace {

using namespace sm100;

constexpr int kTcThreads = 256;
constexpr int kN = 128, kP = 64, kHalf = 64;

template <int R>
struct TcCfg {
    static constexpr int Q = 64 / R;                        // tokens per chunk
    static constexpr int TPL = Q >= 32 ? Q / 32 : 1;        // tokens per lane (rotation)
    static constexpr int PPL = (Q / 4) / TPL;               // pairs per lane (rotation)
    static constexpr int LPT = 8 / PPL;                     // lanes per token group
    static_assert(LPT * (Q / TPL) == 32, "rotation lane mapping");
};

// smem byte layout (after 1024-byte alignment)
constexpr uint32_t OFF_X = 0;           // X chunk, 64 rows x 128 B, swizzled (TMA)
constexpr uint32_t OFF_XP = 8192;       // X' = diag(dw) X
constexpr uint32_t OFF_B = 16384;       // Bbar, 2 slabs of 64 rows x 128 B
constexpr uint32_t OFF_C = 32768;       // Cbar, 2 slabs
constexpr uint32_t OFF_P = 49152;       // P = S o M, 64 rows x 128 B
constexpr uint32_t OFF_H = 57344;       // H0 bf16, 128 rows x 128 B
constexpr uint32_t OFF_F = 73728;       // fp32 scratch
// fp32 scratch (float offsets from OFF_F)
constexpr int F_CUM = 0, F_GAM = 64, F_W = 128, F_ECUM = 192, F_DW = 256, F_DT = 320,
              F_RSB = 384, F_RSC = 448, F_MISC = 512, F_BIAS = 576;
// F_BIAS: bias_B [R][128] then bias_C [R][128]; then prev-token fold scratch
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t T_S = 0, T_YO = 64, T_YD = 128, T_DH = 192;

__host__ __device__ constexpr uint32_t tc_smem_bytes(int R) {
    return OFF_F + 4u * (F_BIAS + 2 * R * 128 + R * 128 + R * 64) + 1024u;
}

// Cody-Waite reduction of x by 2*pi (Cody & Waite, "Software Manual for the Elementary
// Functions", 1980) into [-pi, pi], then the hardware sine/cosine. Absolute error ~1e-6 for
// |x| < 1e4, far below the bf16 rounding of the rotated operands.
__device__ __forceinline__ void sincos_2pi_reduced(float x, float* s, float* c) {
    constexpr float kInv2Pi = 0.15915494309189535f;
    constexpr float k2PiHi = 6.28125f;                  // exactly representable head of 2*pi
    constexpr float k2PiLo = 1.9353071795864769e-3f;    // 2*pi - 6.28125
    const float k = rintf(x * kInv2Pi);
    float r = fmaf(-k, k2PiHi, x);
    r = fmaf(-k, k2PiLo, r);
    __sincosf(r, s, c);
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&v);
}

// Loads PPL consecutive bf16 as floats (PPL in {2, 4, 8}).
template <int PPL>
__device__ __forceinline__ void ld_bf16(const __nv_bfloat16* src, float (&v)[PPL]) {
    if constexpr (PPL == 8) {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(src));
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(&w[i]);
            v[2 * i] = __low2float(h);
            v[2 * i + 1] = __high2float(h);
        }
    } else if constexpr (PPL == 4) {
        const uint2 u = __ldg(reinterpret_cast<const uint2*>(src));
        const uint32_t w[2] = {u.x, u.y};
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(&w[i]);
            v[2 * i] = __low2float(h);
            v[2 * i + 1] = __high2float(h);
        }
    } else {
        const uint32_t u = __ldg(reinterpret_cast<const unsigned int*>(src));
        const __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(&u);
        v[0] = __low2float(h);
        v[1] = __high2float(h);
    }
}

template <int PPL>
__device__ __forceinline__ void st_bf16_smem(uint8_t* dst, const float (&v)[PPL]) {
    if constexpr (PPL == 8) {
        uint4 u;
        u.x = pack_bf16(v[0], v[1]); u.y = pack_bf16(v[2], v[3]);
        u.z = pack_bf16(v[4], v[5]); u.w = pack_bf16(v[6], v[7]);
        *reinterpret_cast<uint4*>(dst) = u;
    } else if constexpr (PPL == 4) {
        uint2 u;
        u.x = pack_bf16(v[0], v[1]); u.y = pack_bf16(v[2], v[3]);
        *reinterpret_cast<uint2*>(dst) = u;
    } else {
        *reinterpret_cast<uint32_t*>(dst) = pack_bf16(v[0], v[1]);
    }
}

__device__ __forceinline__ void set_status(int32_t* status, int code) {
    if (status) atomicExch(status, code);
}

template <int R>
__global__ void __launch_bounds__(kTcThreads, 2)
scan_tc_kernel(const ScanParams p, const __grid_constant__ CUtensorMap tmx) {
    using Cfg = TcCfg<R>;
    constexpr int Q = Cfg::Q, TPL = Cfg::TPL, PPL = Cfg::PPL, LPT = Cfg::LPT;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    float* sf = reinterpret_cast<float*>(sm + OFF_F);
    float* s_biasB = sf + F_BIAS;
    float* s_biasC = s_biasB + R * kN;
    float* s_fold = s_biasC + R * kN;     // [R][128] Bbar of the stored previous token
    float* s_foldx = s_fold + R * kN;     // [R][64]  its x
    __shared__ uint64_t bar_x, bar_m1, bar_m2;
    __shared__ uint32_t tslot;
    __shared__ int s_abort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q4 = warp & 3, wh = warp >> 2;  // TMEM subpartition, column half
    const int64_t u = blockIdx.x;
    const int64_t bb = u / p.H, hh = u % p.H, g = hh / (p.H / p.G);
    const int64_t L = p.L;
    const __nv_bfloat16* xg = static_cast<const __nv_bfloat16*>(p.x);
    const __nv_bfloat16* Bg = static_cast<const __nv_bfloat16*>(p.B);
    const __nv_bfloat16* Cg = static_cast<const __nv_bfloat16*>(p.C);
    const __nv_bfloat16* thg = static_cast<const __nv_bfloat16*>(p.theta);
    __nv_bfloat16* yg = static_cast<__nv_bfloat16*>(p.y);
    auto sidx = [&](int64_t t) { return (bb * L + t) * p.H + hh; };

    // ---------------- setup ----------------
    if (tid == 0) {
        mbar_init(&bar_x, 1);
        mbar_init(&bar_m1, 1);
        mbar_init(&bar_m2, 1);
        fence_mbar_init();
        s_abort = 0;
    }
    if (warp == 0) tmem_alloc(&tslot, kTmemCols);
    for (int i = tid; i < R * kN; i += kTcThreads) {
        s_biasB[i] = p.Bbias ? p.Bbias[hh * R * kN + i] : 0.f;
        s_biasC[i] = p.Cbias ? p.Cbias[hh * R * kN + i] : 0.f;
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = tslot;

    // state rows owned by this thread: n = 32*q4 + lane, columns [32*wh, 32*wh + 32)
    const int nrow = 32 * q4 + lane;
    float hreg[32];
    if (p.h0) {
        const float4* src = reinterpret_cast<const float4*>(p.h0 + (u * kN + nrow) * kP + 32 * wh);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float4 v = src[j];
            hreg[4 * j] = v.x; hreg[4 * j + 1] = v.y; hreg[4 * j + 2] = v.z; hreg[4 * j + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) hreg[j] = 0.f;
    }

    // rotation lane mapping: warp -> 8 pairs, lane -> (token group, pair subgroup)
    const int tg = lane / LPT, ps = lane % LPT;
    const int pp0 = 8 * warp + ps * PPL;  // first pair of this lane
    float carry[PPL];
#pragma unroll
    for (int j = 0; j < PPL; ++j) carry[j] = p.phi0 ? p.phi0[u * kHalf + pp0 + j] : 0.f;

    // ---- fold the stored previous token into the primed state ----
    if (p.h0 && L > 0) {
        const __nv_bfloat16* pB = static_cast<const __nv_bfloat16*>(p.prevB0) + u * R * kN;
        const __nv_bfloat16* px = static_cast<const __nv_bfloat16*>(p.prevx0) + u * R * kP;
        if (warp < R) {  // RMS scale of the stored raw B, one warp per rank
            float ss = 0.f;
            for (int n = lane; n < kN; n += 32) {
                const float v = __bfloat162float(pB[warp * kN + n]);
                ss += v * v;
            }
            ss = warp_sum(ss);
            if (lane == 0) sf[F_MISC + 8 + warp] = p.bc_norm ? rsqrtf(ss / kN + p.eps) : 1.f;
        }
        for (int i = tid; i < R * kP; i += kTcThreads) s_foldx[i] = __bfloat162float(px[i]);
        __syncthreads();
        for (int k = tid; k < R * kHalf; k += kTcThreads) {
            const int r = k / kHalf, i = k % kHalf;
            float sn, cs;
            sincosf(p.phi0[u * kHalf + i], &sn, &cs);
            const float rs = sf[F_MISC + 8 + r];
            const float u0 = __bfloat162float(pB[r * kN + i]) * rs + s_biasB[r * kN + i];
            const float u1 = __bfloat162float(pB[r * kN + i + kHalf]) * rs + s_biasB[r * kN + i + kHalf];
            s_fold[r * kN + i] = u0 * cs + u1 * sn;
            s_fold[r * kN + i + kHalf] = u1 * cs - u0 * sn;
        }
        __syncthreads();
        const float f = (1.f - p.lam[sidx(0)]) * p.dt[sidx(0)];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            float acc = 0.f;
#pragma unroll
            for (int r = 0; r < R; ++r) acc = fmaf(s_fold[r * kN + nrow], s_foldx[r * kP + 32 * wh + j], acc);
            hreg[j] = fmaf(f, acc, hreg[j]);
        }
    }

    const uint32_t aB = smem_u32(sm + OFF_B), aC = smem_u32(sm + OFF_C);
    const uint32_t aX = smem_u32(sm + OFF_X), aXP = smem_u32(sm + OFF_XP);
    const uint32_t aP = smem_u32(sm + OFF_P), aH = smem_u32(sm + OFF_H);
    const uint32_t id_s = idesc_bf16(64, 64, false, false);   // S  = C . B^T
    const uint32_t id_yo = idesc_bf16(64, 64, false, true);   // Yo = C . H
    const uint32_t id_dh = idesc_bf16(128, 64, true, true);   // dH = B^T . X'
    const uint32_t id_yd = idesc_bf16(64, 64, false, true);   // Yd = P . X

    const int64_t nchunks = (L + Q - 1) / Q;
    for (int64_t c = 0; c < nchunks; ++c) {
        const int64_t c0 = c * Q;
        const int T = static_cast<int>((L - c0) < Q ? (L - c0) : Q);
        const uint32_t par = static_cast<uint32_t>(c & 1);

        // ---- A. TMA of X, chunk scalars, norms ----
        if (tid == 0) {
            mbar_arrive_expect_tx(&bar_x, 64 * 128);
            tma_load_5d(sm + OFF_X, &tmx, &bar_x, 0, 0, static_cast<int>(hh), static_cast<int>(c0),
                        static_cast<int>(bb));
        }
        __syncwarp();
        if (warp == 0) {
            // token t = lane (+32): a = dt*A, inclusive scan -> cum; gamma, w
            float a[2], d[2], ga[2], w[2];
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int t = lane + 32 * k;
                a[k] = d[k] = ga[k] = w[k] = 0.f;
                if (t < T) {
                    const int64_t si = sidx(c0 + t);
                    const float dd = p.dt[si], lm = p.lam[si];
                    d[k] = dd;
                    a[k] = dd * p.A[si];
                    ga[k] = lm * dd;
                    w[k] = ga[k];
                    if (c0 + t + 1 < L) {
                        const int64_t sn = sidx(c0 + t + 1);
                        w[k] += (1.f - p.lam[sn]) * p.dt[sn];
                    }
                }
            }
            float c0s = warp_inclusive_scan(a[0]);
            const float tot0 = __shfl_sync(0xffffffffu, c0s, 31);
            float c1s = warp_inclusive_scan(a[1]) + tot0;
            const float cum_end = __shfl_sync(0xffffffffu, (T - 1) < 32 ? c0s : c1s, (T - 1) & 31);
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int t = lane + 32 * k;
                if (t < 64) {
                    const float cm = (t < T) ? (k ? c1s : c0s) : cum_end;
                    sf[F_CUM + t] = cm;
                    sf[F_GAM + t] = ga[k];
                    sf[F_W + t] = w[k];
                    sf[F_ECUM + t] = __expf(cm);
                    sf[F_DW + t] = (t < T) ? __expf(cum_end - cm) * w[k] : 0.f;
                    sf[F_DT + t] = d[k];
                }
            }
            if (lane == 0) sf[F_MISC] = __expf(cum_end);
        }
        {
            // RMS scales: 2 threads per (row, tensor)
            const int pr = tid >> 1, half = tid & 1;
            const int tensor = pr >> 6, row = pr & 63;
            const int t = row / R, r = row % R;
            float ss = 0.f;
            if (t < T) {
                const __nv_bfloat16* src = (tensor ? Cg : Bg) +
                    (((bb * L + c0 + t) * p.G + g) * R + r) * kN + half * 64;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    float v[8];
                    ld_bf16<8>(src + 8 * j, v);
#pragma unroll
                    for (int e = 0; e < 8; ++e) ss = fmaf(v[e], v[e], ss);
                }
            }
            ss += __shfl_xor_sync(0xffffffffu, ss, 1);
            if (half == 0) sf[(tensor ? F_RSC : F_RSB) + row] = p.bc_norm ? rsqrtf(ss / kN + p.eps) : 1.f;
        }
        __syncthreads();

        // ---- B. cumulative angle (warp scan over tokens) and rotation into Bbar / Cbar ----
        {
            float inc[TPL][PPL];
#pragma unroll
            for (int k = 0; k < TPL; ++k) {
                const int t = tg * TPL + k;
                float th[PPL];
                if (t < T) {
                    ld_bf16<PPL>(thg + sidx(c0 + t) * kHalf + pp0, th);
                } else {
#pragma unroll
                    for (int j = 0; j < PPL; ++j) th[j] = 0.f;
                }
                const float dd = sf[F_DT + t];
#pragma unroll
                for (int j = 0; j < PPL; ++j) inc[k][j] = dd * th[j] + (k ? inc[k - 1][j] : 0.f);
            }
            float incl[PPL], base[PPL];
#pragma unroll
            for (int j = 0; j < PPL; ++j) incl[j] = inc[TPL - 1][j];
#pragma unroll
            for (int off = LPT; off < 32; off <<= 1) {
#pragma unroll
                for (int j = 0; j < PPL; ++j) {
                    const float v = __shfl_up_sync(0xffffffffu, incl[j], off);
                    if (lane >= off) incl[j] += v;
                }
            }
#pragma unroll
            for (int j = 0; j < PPL; ++j) {
                base[j] = carry[j] + incl[j] - inc[TPL - 1][j];
                carry[j] += __shfl_sync(0xffffffffu, incl[j], 32 - LPT + ps);
            }
#pragma unroll
            for (int k = 0; k < TPL; ++k) {
                const int t = tg * TPL + k;
                float cs[PPL], sn[PPL];
#pragma unroll
                for (int j = 0; j < PPL; ++j) sincos_2pi_reduced(base[j] + inc[k][j], &sn[j], &cs[j]);
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const int row = t * R + r;
                    float ob0[PPL], ob1[PPL], oc0[PPL], oc1[PPL];
                    if (t < T) {
                        const int64_t gi = (((bb * L + c0 + t) * p.G + g) * R + r) * kN + pp0;
                        float b0[PPL], b1[PPL], cc0[PPL], cc1[PPL];
                        ld_bf16<PPL>(Bg + gi, b0);
                        ld_bf16<PPL>(Bg + gi + kHalf, b1);
                        ld_bf16<PPL>(Cg + gi, cc0);
                        ld_bf16<PPL>(Cg + gi + kHalf, cc1);
                        const float rb = sf[F_RSB + row], rc = sf[F_RSC + row];
#pragma unroll
                        for (int j = 0; j < PPL; ++j) {
                            const int n = pp0 + j;
                            float u0 = fmaf(b0[j], rb, s_biasB[r * kN + n]);
                            float u1 = fmaf(b1[j], rb, s_biasB[r * kN + n + kHalf]);
                            ob0[j] = fmaf(u0, cs[j], u1 * sn[j]);
                            ob1[j] = fmaf(u1, cs[j], -u0 * sn[j]);
                            u0 = fmaf(cc0[j], rc, s_biasC[r * kN + n]);
                            u1 = fmaf(cc1[j], rc, s_biasC[r * kN + n + kHalf]);
                            oc0[j] = fmaf(u0, cs[j], u1 * sn[j]);
                            oc1[j] = fmaf(u1, cs[j], -u0 * sn[j]);
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < PPL; ++j) ob0[j] = ob1[j] = oc0[j] = oc1[j] = 0.f;
                    }
                    const uint32_t o = swz128(row, pp0);
                    st_bf16_smem<PPL>(sm + OFF_B + o, ob0);
                    st_bf16_smem<PPL>(sm + OFF_B + 8192 + o, ob1);
                    st_bf16_smem<PPL>(sm + OFF_C + o, oc0);
                    st_bf16_smem<PPL>(sm + OFF_C + 8192 + o, oc1);
                }
            }
        }
        // H0 (bf16) as the Yo operand: row nrow, columns [32 wh, 32 wh + 32)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint4 v;
            v.x = pack_bf16(hreg[8 * i + 0], hreg[8 * i + 1]);
            v.y = pack_bf16(hreg[8 * i + 2], hreg[8 * i + 3]);
            v.z = pack_bf16(hreg[8 * i + 4], hreg[8 * i + 5]);
            v.w = pack_bf16(hreg[8 * i + 6], hreg[8 * i + 7]);
            *reinterpret_cast<uint4*>(sm + OFF_H + swz128(nrow, 32 * wh + 8 * i)) = v;
        }

        // ---- C. X' = diag(dw) X once X has landed ----
        if (!mbar_wait(&bar_x, par)) {
            if (lane == 0) s_abort = 1;
        }
        for (int e = tid; e < 64 * 8; e += kTcThreads) {
            const int row = e >> 3, ch = e & 7;
            const float sc = sf[F_DW + row / R];
            const uint32_t o = static_cast<uint32_t>(row) * 128u + (static_cast<uint32_t>(ch) << 4);
            uint4 v = *reinterpret_cast<const uint4*>(sm + OFF_X + o);
            uint32_t wds[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                __nv_bfloat162 h2 = *reinterpret_cast<__nv_bfloat162*>(&wds[i]);
                wds[i] = pack_bf16(__low2float(h2) * sc, __high2float(h2) * sc);
            }
            *reinterpret_cast<uint4*>(sm + OFF_XP + o) = make_uint4(wds[0], wds[1], wds[2], wds[3]);
        }
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();
        fence_after_sync();
        if (s_abort) break;

        // ---- D. S, Yo, dH ----
        if (tid == 0) {
#pragma unroll
            for (int k = 0; k < 8; ++k)
                mma_bf16(tmem + T_S, sdesc_kmajor(aC, k, 8192), sdesc_kmajor(aB, k, 8192), id_s, k > 0);
#pragma unroll
            for (int k = 0; k < 8; ++k)
                mma_bf16(tmem + T_YO, sdesc_kmajor(aC, k, 8192), sdesc_mnmajor(aH, k, 16384), id_yo, k > 0);
#pragma unroll
            for (int k = 0; k < 4; ++k)
                mma_bf16(tmem + T_DH, sdesc_mnmajor(aB, k, 8192), sdesc_mnmajor(aXP, k, 8192), id_dh, k > 0);
            mma_commit(smem_u32(&bar_m1));
        }
        __syncwarp();
        if (!mbar_wait(&bar_m1, par)) {
            if (lane == 0) s_abort = 1;
        }
        fence_after_sync();

        // ---- E. P = S o M  and  H1 = e^{cum_end} H0 + dH ----
        {
            float s[16];
            const uint32_t ta = tmem + ((32u * q4) << 16) + T_S + 16u * wh;
            tmem_ld_16x32bx2_x16(ta, s);
            tmem_wait_ld();
            const int trow = 16 * q4 + (lane & 15);
            const int col0 = 16 * wh + ((lane >> 4) ? 32 : 0);
            const int t = trow / R;
            const float cum_t = sf[F_CUM + t], gam_t = sf[F_GAM + t];
            float pv[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int sidx2 = (col0 + j) / R;
                float m = 0.f;
                if (sidx2 < t) m = __expf(cum_t - sf[F_CUM + sidx2]) * sf[F_W + sidx2];
                else if (sidx2 == t) m = gam_t;
                pv[j] = s[j] * m;
            }
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                uint4 v;
                v.x = pack_bf16(pv[8 * i + 0], pv[8 * i + 1]);
                v.y = pack_bf16(pv[8 * i + 2], pv[8 * i + 3]);
                v.z = pack_bf16(pv[8 * i + 4], pv[8 * i + 5]);
                v.w = pack_bf16(pv[8 * i + 6], pv[8 * i + 7]);
                *reinterpret_cast<uint4*>(sm + OFF_P + swz128(trow, col0 + 8 * i)) = v;
            }
        }
        {
            const float eend = sf[F_MISC];
            const uint32_t ta = tmem + ((32u * q4) << 16) + T_DH + 32u * wh;
            float d0[16], d1[16];
            tmem_ld_32x32b_x16(ta, d0);
            tmem_ld_32x32b_x16(ta + 16, d1);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                hreg[j] = fmaf(eend, hreg[j], d0[j]);
                hreg[16 + j] = fmaf(eend, hreg[16 + j], d1[j]);
            }
        }
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();
        fence_after_sync();
        if (s_abort) break;

        // ---- F. Yd = P X ----
        if (tid == 0) {
#pragma unroll
            for (int k = 0; k < 4; ++k)
                mma_bf16(tmem + T_YD, sdesc_kmajor(aP, k, 8192), sdesc_mnmajor(aX, k, 8192), id_yd, k > 0);
            mma_commit(smem_u32(&bar_m2));
        }
        __syncwarp();
        if (!mbar_wait(&bar_m2, par)) {
            if (lane == 0) s_abort = 1;
        }
        fence_after_sync();

        // ---- G. y = Yd + e^{cum_t} Yo ----
        {
            float yd[16], yo[16];
            const uint32_t lanebase = (32u * q4) << 16;
            tmem_ld_16x32bx2_x16(tmem + lanebase + T_YD + 16u * wh, yd);
            tmem_ld_16x32bx2_x16(tmem + lanebase + T_YO + 16u * wh, yo);
            tmem_wait_ld();
            const int trow = 16 * q4 + (lane & 15);
            const int col0 = 16 * wh + ((lane >> 4) ? 32 : 0);
            const int t = trow / R, r = trow % R;
            if (t < T) {
                const float e = sf[F_ECUM + t];
                __nv_bfloat16* dst = yg + (((bb * L + c0 + t) * p.H + hh) * R + r) * kP + col0;
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    uint4 v;
                    v.x = pack_bf16(fmaf(e, yo[8 * i + 0], yd[8 * i + 0]), fmaf(e, yo[8 * i + 1], yd[8 * i + 1]));
                    v.y = pack_bf16(fmaf(e, yo[8 * i + 2], yd[8 * i + 2]), fmaf(e, yo[8 * i + 3], yd[8 * i + 3]));
                    v.z = pack_bf16(fmaf(e, yo[8 * i + 4], yd[8 * i + 4]), fmaf(e, yo[8 * i + 5], yd[8 * i + 5]));
                    v.w = pack_bf16(fmaf(e, yo[8 * i + 6], yd[8 * i + 6]), fmaf(e, yo[8 * i + 7], yd[8 * i + 7]));
                    *reinterpret_cast<uint4*>(dst + 8 * i) = v;
                }
            }
        }
        fence_before_sync();
        __syncthreads();
        fence_after_sync();
        if (s_abort) break;
    }

    // ---------------- final state ----------------
    if (!s_abort) {
        if (p.h1) {
            float4* dst = reinterpret_cast<float4*>(p.h1 + (u * kN + nrow) * kP + 32 * wh);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                dst[j] = make_float4(hreg[4 * j], hreg[4 * j + 1], hreg[4 * j + 2], hreg[4 * j + 3]);
        }
        if (p.phi1 && tg == 0) {
#pragma unroll
            for (int j = 0; j < PPL; ++j) p.phi1[u * kHalf + pp0 + j] = carry[j];
        }
        if (L > 0) {
            if (p.prevB1) {
                __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.prevB1) + u * R * kN;
                const __nv_bfloat16* src = Bg + ((bb * L + L - 1) * p.G + g) * R * kN;
                for (int e = tid; e < R * kN; e += kTcThreads) dst[e] = src[e];
            }
            if (p.prevx1) {
                __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.prevx1) + u * R * kP;
                const __nv_bfloat16* src = xg + ((bb * L + L - 1) * p.H + hh) * R * kP;
                for (int e = tid; e < R * kP; e += kTcThreads) dst[e] = src[e];
            }
        }
    } else if (tid == 0) {
        set_status(p.status, 1);
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }
    return fn;
}

}  // namespace

bool tc_scan_supported(const ScanParams& p, bool bf16) {
    return bf16 && p.N == kN && p.P == kP && p.Q * p.R == 64 &&
           (p.R == 1 || p.R == 2 || p.R == 4 || p.R == 8) && p.L <= 0x7fffffffLL;
}

template <int R>
static cudaError_t launch_tc_t(const ScanParams& p, cudaStream_t s) {
    auto enc = get_encode();
    if (!enc) return cudaErrorNotSupported;
    // x viewed as 5D [b][L][H][R][P] (innermost first for the map), box (P, R, 1, Q, 1)
    CUtensorMap map;
    const cuuint64_t dims[5] = {static_cast<cuuint64_t>(kP), static_cast<cuuint64_t>(R),
                                static_cast<cuuint64_t>(p.H), static_cast<cuuint64_t>(p.L),
                                static_cast<cuuint64_t>(p.b)};
    const cuuint64_t strides[4] = {static_cast<cuuint64_t>(kP) * 2,
                                   static_cast<cuuint64_t>(R * kP) * 2,
                                   static_cast<cuuint64_t>(p.H * R * kP) * 2,
                                   static_cast<cuuint64_t>(p.L * p.H * R * kP) * 2};
    const cuuint32_t box[5] = {static_cast<cuuint32_t>(kP), static_cast<cuuint32_t>(R), 1u,
                               static_cast<cuuint32_t>(64 / R), 1u};
    const cuuint32_t es[5] = {1, 1, 1, 1, 1};
    CUresult cr = enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(p.x), dims,
                      strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return cudaErrorInvalidValue;
    const uint32_t smem = tc_smem_bytes(R);
    auto k = scan_tc_kernel<R>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    k<<<static_cast<unsigned>(p.b * p.H), kTcThreads, smem, s>>>(p, map);
    return cudaGetLastError();
}

cudaError_t launch_scan_tc(const ScanParams& p, cudaStream_t s) {
    if (p.b * p.H == 0) return cudaSuccess;
    switch (p.R) {
        case 1: return launch_tc_t<1>(p, s);
        case 2: return launch_tc_t<2>(p, s);
        case 4: return launch_tc_t<4>(p, s);
        case 8: return launch_tc_t<8>(p, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace m3
