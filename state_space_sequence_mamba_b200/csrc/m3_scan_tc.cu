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
// Data flow per CTA (one (batch, head) unit, 8 warps, two CTAs per SM): every per-chunk
// input of the next chunk (X, theta, dt, A, lam) is fetched by TMA into the other half of a
// double buffer while the current chunk computes; X lands in the 128-byte swizzled layout the
// MMA reads. B and C are shared by all heads, so their rows come from L2; their RMS scales are
// computed once per token by a small pre-pass instead of once per head. Normalisation, bias
// and rotation run on the CUDA cores straight into swizzled bf16 operand tiles. The fp32
// state lives in registers (row n of the state in lane n of the TMEM datapath, matching the
// dH accumulator) and is rounded to bf16 only as the Yo operand. All waits are bounded; a
// timeout sets the status word and the CTA exits cleanly.
#include <algorithm>
#include <cstdlib>

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

__host__ __device__ constexpr uint32_t round_up(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

template <int R>
struct TcCfg {
    static constexpr int Q = 64 / R;                        // tokens per chunk
    static constexpr int TPS = Q / 8;                       // tokens per warp (rotation)
    static_assert(TPS * 8 == Q, "one token segment per warp");
    // shared-memory byte layout after 1024-byte alignment
    static constexpr uint32_t X0 = 0, X1 = 8192;             // X chunk (TMA, swizzled), x2
    static constexpr uint32_t XP = 16384;                    // X' = diag(dw) X, then P = S o M
    static constexpr uint32_t OB = 24576;                    // Bbar, 2 slabs of 64 x 128 B
    static constexpr uint32_t OC = 40960;                    // raw C, rotated in place to Cbar
    static constexpr uint32_t OH = 57344;                    // H0 bf16, 128 x 128 B
    static constexpr uint32_t RB = 73728;                    // raw B of the chunk (TMA)
    static constexpr uint32_t TH_BYTES = round_up(Q * 128, 1024);
    static constexpr uint32_t TH = 90112;                    // theta (TMA, swizzled)
    static constexpr uint32_t SC_ONE = (Q + 1) * 16;                // [Q+1 tokens][4 heads] fp32
    static constexpr uint32_t SC_SLOT = round_up(SC_ONE, 128);      // 128-byte aligned slots
    static constexpr uint32_t SC_BYTES = 3 * SC_SLOT;
    static constexpr uint32_t SC0 = TH + TH_BYTES, SC1 = SC0 + SC_BYTES;  // dt, A, lam boxes
    static constexpr uint32_t ORS = SC1 + SC_BYTES;                 // RMS scales, 64 x float2
    static constexpr uint32_t OF = ORS + 512;                       // fp32 scratch
    static constexpr uint32_t B_TX = 2 * 8192;                      // raw B: two slabs
    static constexpr uint32_t C_TX = 2 * 8192;                      // raw C: two slabs
    static constexpr uint32_t X_TX = 8192;                          // bytes of one X box
    static constexpr uint32_t TH_TX = Q * 128;                      // theta box
    static constexpr uint32_t SC_TX = 3 * SC_ONE;                   // dt, A, lam boxes
};
// fp32 scratch (float offsets): two blocks of chunk scalars (by chunk parity), the angle
// totals of the eight token segments, then the bf16 biases
constexpr int F_CUM = 0, F_GAM = 64, F_W = 128, F_ECUM = 192, F_DW = 256, F_DT = 320,
              F_EROW = 384, F_ECOL = 448,  // tile factors: [64], column blocks 1..3 x [64]
              F_MISC = 640,                // e^{cum_end}
              F_BLK = 656;
constexpr int F_SEG = 2 * F_BLK;           // [8 segments][32 lanes] float2
constexpr int F_BIAS = F_SEG + 512;        // bias_B [R][128] fp32, bias_C [R][128] fp32
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t T_S = 0, T_YO = 64, T_YD = 128, T_DH = 192;
// One state slot in the workspace (floats): h [N][P], the angle [N/2], a segment's summed
// log-decay, padding to a multiple of 16 bytes.
constexpr int kSegStride = kN * kP + kHalf + 4;

template <int R>
__host__ __device__ constexpr uint32_t tc_smem_bytes() {
    return TcCfg<R>::OF + 4u * F_BIAS + 4u * 2 * R * kN + 1024u;
}

// 2^x by the hardware approximation (relative error ~2^-22), x <= 0 here.
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&v);
}

// (low, high) bf16 halves of a word as exact fp32, and two floats rounded to a bf16 pair
__device__ __forceinline__ float2 bf2_to_f2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}
__device__ __forceinline__ uint32_t f2_to_bf2(float2 v) { return pack_bf16(v.x, v.y); }

__device__ __forceinline__ __nv_bfloat162 as_bf2(uint32_t w) {
    return *reinterpret_cast<const __nv_bfloat162*>(&w);
}
__device__ __forceinline__ uint32_t as_u32(__nv_bfloat162 v) {
    return *reinterpret_cast<const uint32_t*>(&v);
}

struct TcMaps {
    CUtensorMap x, theta, dt, A, lam, B, C;
};

// RMS scale of every B and C row (shared by all heads): one warp per row of N = 128. Rows
// (b, l, g, r) are written to out[((b * G + g) * Lpad + l) * R + r] so that the rows of one
// chunk of one group are contiguous (one bulk copy per chunk); Lpad rounds L up to chunks.
__global__ void __launch_bounds__(256) rms_scale_kernel(const __nv_bfloat16* __restrict__ B,
                                                        const __nv_bfloat16* __restrict__ C,
                                                        int64_t rows, int64_t L, int64_t G,
                                                        int64_t R, int64_t Lpad, float eps,
                                                        float2* __restrict__ out) {
    grid_dep_launch_dependents();   // the scan's set-up may overlap this kernel
    const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) {
        // the rows past the sequence end in the last chunk: zero scales (their B and C rows are
        // zero-filled loads, so the scaled value is 0 whatever the workspace held before)
        const int64_t pr = row - rows, pad = Lpad - L;
        if (lane == 0 && pad > 0 && pr < (rows / (L * G * R)) * G * pad * R) {
            const int64_t r = pr % R, g = (pr / R) % G, l = L + (pr / (R * G)) % pad;
            const int64_t b = pr / (R * G * pad);
            out[((b * G + g) * Lpad + l) * R + r] = make_float2(0.f, 0.f);
        }
        return;
    }
    const int64_t r = row % R, g = (row / R) % G, l = (row / (R * G)) % L, b = row / (R * G * L);
    const int64_t orow = ((b * G + g) * Lpad + l) * R + r;
    const uint2 ub = __ldg(reinterpret_cast<const uint2*>(B + row * kN) + lane);
    const uint2 uc = __ldg(reinterpret_cast<const uint2*>(C + row * kN) + lane);
    float sb = 0.f, sc = 0.f;
    const uint32_t wb[2] = {ub.x, ub.y}, wc[2] = {uc.x, uc.y};
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const float b0 = __uint_as_float(wb[i] << 16), b1 = __uint_as_float(wb[i] & 0xFFFF0000u);
        const float c0 = __uint_as_float(wc[i] << 16), c1 = __uint_as_float(wc[i] & 0xFFFF0000u);
        sb = fmaf(b0, b0, fmaf(b1, b1, sb));
        sc = fmaf(c0, c0, fmaf(c1, c1, sc));
    }
    sb = warp_sum(sb);
    sc = warp_sum(sc);
    if (lane == 0) out[orow] = make_float2(rsqrtf(sb / kN + eps), rsqrtf(sc / kN + eps));
}

// The sequence-parallel form for few long sequences: the sequence of every unit is cut into
// nseg segments of seg_chunks chunks (the last may be shorter). A state-only pass computes each
// segment's end state but the last's; the full pass then runs every segment at once from the
// state at its start, which it assembles from those end states. nseg = 1 is the plain scan.
// Per unit, slots 0 .. nseg-2 hold the segments' end states and slot nseg-1 the primed initial
// state (the given state with the stored token folded in): the full pass reads no caller state,
// so the final state may overwrite the initial one while other segments still run.
struct SegArgs {
    int seg_chunks = 0, nseg = 1;
    float* st = nullptr;   // [units][nseg][kSegStride]
    // m3_scan_state in one segment: the end state goes to the caller's buffers instead:
    // h [units][N][P], phi [units][N/2], the summed log-decay [units]
    float* out_h = nullptr;
    float* out_phi = nullptr;
    float* out_lam = nullptr;
    // the state-only pass keeps segment 0's primed initial state in slot nseg-1 for the full
    // pass (not when every segment's end state is wanted, as for m3_scan_state)
    bool save_init = true;
    // one segment, for the backward: per unit and chunk, e^{cum_0} H0' as bf16 in the swizzled
    // [n][p] operand layout (16384 bytes) and the angle before the chunk (64 floats)
    uint8_t* chunk_h = nullptr;
    float* chunk_phi = nullptr;
};

// One CTA per (unit, segment), CTA index = segment * units + unit. kStateOnly: the segment's
// end state only (no C, S, Yo, Yd, y); segment 0 starts from the given initial state in the
// true angle frame, later segments from zero in their own frame (angle 0 at their start).
// kRaw: dt and lam arrive raw (m3_dims.flags) and the chunk scalars apply softplus / sigmoid.
template <int R, bool kStateOnly, bool kRaw>
__global__ void __launch_bounds__(kTcThreads, 2)
scan_tc_kernel(const ScanParams p, const __grid_constant__ TcMaps maps, const float2* __restrict__ rsrow,
               const SegArgs sa) {
    using Cfg = TcCfg<R>;
    constexpr int Q = Cfg::Q, TPS = Cfg::TPS;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    float* sf = reinterpret_cast<float*>(sm + Cfg::OF);   // two blocks of chunk scalars
    float2* s_seg = reinterpret_cast<float2*>(sf + F_SEG);
    float* s_biasB = sf + F_BIAS;              // [R][128]
    float* s_biasC = s_biasB + R * kN;
    // set-up only: the stored previous token's Bbar and x, in the H0 operand buffer
    float* s_fold = reinterpret_cast<float*>(sm + Cfg::OH);   // [R][128]
    float* s_foldx = s_fold + R * kN;                          // [R][64]
    __shared__ uint64_t bar_x[2], bar_sc[2], bar_th, bar_b, bar_c, bar_yo, bar_s, bar_dh, bar_m2;
    __shared__ uint32_t tslot;
    __shared__ int s_abort;
    // async work thread 0 has started, for draining it if a wait gives up: last X and scalar
    // box chunk issued; theta, raw B, raw C loads issued; MMA groups (Yo, S, dH) and Yd committed
    __shared__ int s_issued[7];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q4 = warp & 3, wh = warp >> 2;  // TMEM subpartition, column half
    // One elected lane of this warp issues every TMA copy and MMA: its share of the masking
    // (row block 0, column blocks 1 and 3) is all zeros.
    constexpr int kIssueWarp = 4;
    const int units32 = static_cast<int>(p.b * p.H);   // < 2^31 (one CTA per unit and segment)
    const int kseg = static_cast<int>(blockIdx.x) / units32;
    const int64_t u = static_cast<int>(blockIdx.x) - kseg * units32;
    const int64_t bb = u / p.H, hh = u % p.H, g = hh / (p.H / p.G);
    const int hc = static_cast<int>(hh & 3);  // column of this head in the scalar boxes
    const int L = static_cast<int>(p.L);
    const int H = static_cast<int>(p.H), G = static_cast<int>(p.G);
    // Per-unit base pointers; offsets below fit in 32 bits (checked on the host).
    const __nv_bfloat16* Bu = static_cast<const __nv_bfloat16*>(p.B) + (bb * p.L * G + g) * R * kN;
    const int Lpad = ((L + Q - 1) / Q) * Q;
    const float2* rsu = rsrow ? rsrow + (bb * G + g) * static_cast<int64_t>(Lpad) * R : nullptr;
    const __nv_bfloat16* xu = static_cast<const __nv_bfloat16*>(p.x) + (bb * p.L * H + hh) * R * kP;
    __nv_bfloat16* yu = static_cast<__nv_bfloat16*>(p.y) + (bb * p.L * H + hh) * R * kP;
    const int tokB = G * R * kN, tokY = H * R * kP;  // element stride of one token
    // this segment's chunks: global chunks [cb, cb + nchunks); c below is the local index
    const int cb = kseg * sa.seg_chunks;
    const int nchunks = min((L + Q - 1) / Q - cb, sa.seg_chunks);
    const int ib = static_cast<int>(bb), ih = static_cast<int>(hh), ig = static_cast<int>(g);
    float2* s_rs = reinterpret_cast<float2*>(sm + Cfg::ORS);

    // ---- TMA issue (one thread) ----
    auto issue_x = [&](int c) {
        const int st = c & 1;
        mbar_arrive_expect_tx(&bar_x[st], Cfg::X_TX);
        tma_load_5d(sm + (st ? Cfg::X1 : Cfg::X0), &maps.x, &bar_x[st], 0, 0, ih, (cb + c) * Q, ib);
        s_issued[0] = c;
    };
    auto issue_sc = [&](int c) {  // dt, A, lam boxes of chunk c (4 heads, Q + 1 tokens)
        const int st = c & 1;
        mbar_arrive_expect_tx(&bar_sc[st], Cfg::SC_TX);
        uint8_t* sc = sm + (st ? Cfg::SC1 : Cfg::SC0);
        const int h4 = ih & ~3;
        tma_load_3d(sc, &maps.dt, &bar_sc[st], h4, (cb + c) * Q, ib);
        tma_load_3d(sc + Cfg::SC_SLOT, &maps.A, &bar_sc[st], h4, (cb + c) * Q, ib);
        tma_load_3d(sc + 2 * Cfg::SC_SLOT, &maps.lam, &bar_sc[st], h4, (cb + c) * Q, ib);
        s_issued[1] = c;
    };
    auto issue_th = [&](int c) {  // theta of chunk c into the (single) theta buffer
        mbar_arrive_expect_tx(&bar_th, Cfg::TH_TX);
        tma_load_4d(sm + Cfg::TH, &maps.theta, &bar_th, 0, ih, (cb + c) * Q, ib);
        s_issued[2] += 1;
    };
    auto issue_b = [&](int c) {   // raw B rows of chunk c (two 64-column slabs) + RMS scales
        mbar_arrive_expect_tx(&bar_b, Cfg::B_TX + (rsu ? 512u : 0u));
        tma_load_5d(sm + Cfg::RB, &maps.B, &bar_b, 0, 0, ig, (cb + c) * Q, ib);
        tma_load_5d(sm + Cfg::RB + 8192, &maps.B, &bar_b, kHalf, 0, ig, (cb + c) * Q, ib);
        if (rsu) {
            if (c == 0) grid_dep_wait();   // the scales' kernel may still be running
            bulk_load(s_rs, rsu + static_cast<int64_t>(cb + c) * Q * R, 512u, &bar_b);
        }
        s_issued[3] += 1;
    };
    auto issue_c = [&](int c) {   // raw C rows of chunk c straight into the Cbar operand buffer
        mbar_arrive_expect_tx(&bar_c, Cfg::C_TX);
        tma_load_5d(sm + Cfg::OC, &maps.C, &bar_c, 0, 0, ig, (cb + c) * Q, ib);
        tma_load_5d(sm + Cfg::OC + 8192, &maps.C, &bar_c, kHalf, 0, ig, (cb + c) * Q, ib);
        s_issued[4] += 1;
    };
    // Chunk scalars (one full warp, warp 3: its masking share has no diagonal block, so it has
    // the most slack while the MMAs run): cumulative log-decay, gamma, trapezoid weight w, ...; the
    // segment's summed log-decay accumulates in lam_acc
    float lam_acc = 0.f;
    const float dtb = (kRaw && p.dt_bias) ? p.dt_bias[hh] : 0.f;   // only read with M3_DT_SOFTPLUS
    // kRaw: the dt and lam boxes of chunk c arrive raw; threads apply softplus(dt + dt_bias) and
    // sigmoid(lam) in place to this head's column (the box holds 4 heads; the others are not
    // read), real tokens only (positions past the sequence end stay zero), ahead of scalars(c).
    auto raw_box = [&](int c) {
        const int st = c & 1;
        float* sSc = reinterpret_cast<float*>(sm + (st ? Cfg::SC1 : Cfg::SC0));
        const int t0 = (cb + c) * Q;
        constexpr int kCol = Q + 1;   // tokens in the box
        for (int i = tid; i < 2 * kCol; i += kTcThreads) {
            const int t = i < kCol ? i : i - kCol;
            if (t0 + t >= L) continue;
            if (i < kCol) {
                float* d = sSc + t * 4 + hc;
                *d = step_dt<true>(*d, dtb, p.flags);
            } else {
                float* lm = sSc + 2 * Cfg::SC_SLOT / 4 + t * 4 + hc;
                *lm = step_lam<true>(*lm, p.flags);
            }
        }
    };
    auto scalars = [&](int c) {
        const int st = c & 1;
        if (!mbar_wait(&bar_sc[st], (c >> 1) & 1)) {
            if (lane == 0) s_abort = 1;
        }
        const float* sSc = reinterpret_cast<const float*>(sm + (st ? Cfg::SC1 : Cfg::SC0));
        float* blk = sf + st * F_BLK;
        const int T = (L - (cb + c) * Q) < Q ? (L - (cb + c) * Q) : Q;
        constexpr int oA = Cfg::SC_SLOT / 4, oL = 2 * Cfg::SC_SLOT / 4;
        float a[2], d[2], ga[2], w[2];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int t = lane + 32 * k;
            a[k] = d[k] = ga[k] = w[k] = 0.f;
            if (t < T) {
                const float dd = sSc[t * 4 + hc], lm = sSc[oL + t * 4 + hc];
                d[k] = dd;
                a[k] = dd * sSc[oA + t * 4 + hc];
                ga[k] = lm * dd;
                // next token (the box holds Q + 1 tokens, zero-filled past the sequence end)
                w[k] = ga[k] + (1.f - sSc[oL + (t + 1) * 4 + hc]) * sSc[(t + 1) * 4 + hc];
                if constexpr (kRaw) {
                    if (p.flags & 4u) {   // zero-order hold: no previous-token term
                        ga[k] = zoh_gamma(dd, sSc[oA + t * 4 + hc]);
                        w[k] = ga[k];
                    }
                }
            }
        }
        const float c0s = warp_inclusive_scan(a[0]);
        const float tot0 = __shfl_sync(0xffffffffu, c0s, 31);
        const float c1s = warp_inclusive_scan(a[1]) + tot0;
        const float cum_end = __shfl_sync(0xffffffffu, (T - 1) < 32 ? c0s : c1s, (T - 1) & 31);
        if constexpr (kStateOnly) lam_acc += cum_end;
        constexpr float kLog2e = 1.4426950408889634f;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int t = lane + 32 * k;
            const float cm = (t < T) ? (k ? c1s : c0s) : cum_end;
            blk[F_CUM + t] = cm * kLog2e;   // log2-scaled: decays are exp2 of differences
            blk[F_GAM + t] = ga[k];
            blk[F_W + t] = w[k];
            blk[F_ECUM + t] = __expf(cm);
            blk[F_DW + t] = (t < T) ? __expf(cum_end - cm) * w[k] : 0.f;
            blk[F_DT + t] = d[k];
        }
        if (lane == 0) blk[F_MISC] = __expf(cum_end);
        // Tile factors of the decay mask. Rows come in blocks of 16 (16 / R tokens); with t0 the
        // first token of t's block, e^{cum_t - cum_s} = 2^(c2_t - c2_t0) * 2^(c2_t0 - c2_s) for
        // s < t0, both factors <= 1 (cum decreases).
        constexpr int TB = 16 / R;  // tokens per row block
        float c2v[2];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int t = lane + 32 * k;
            c2v[k] = ((t < T) ? (k ? c1s : c0s) : cum_end) * kLog2e;
        }
        float c2blk[4];
#pragma unroll
        for (int qb = 0; qb < 4; ++qb) {
            const int tq = qb * TB;
            c2blk[qb] = __shfl_sync(0xffffffffu, tq < 32 ? c2v[0] : c2v[1], tq & 31);
        }
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int t = lane + 32 * k;
            blk[F_EROW + t] = ex2_approx(c2v[k] - c2blk[t / TB < 4 ? t / TB : 3]);
#pragma unroll
            for (int qb = 1; qb < 4; ++qb)
                blk[F_ECOL + (qb - 1) * 64 + t] = (t < qb * TB) ? ex2_approx(c2blk[qb] - c2v[k]) * w[k] : 0.f;
        }
    };

    // ---------------- setup ----------------
    if (tid == kIssueWarp * 32) {
        mbar_init(&bar_x[0], 1);
        mbar_init(&bar_x[1], 1);
        mbar_init(&bar_sc[0], 1);
        mbar_init(&bar_sc[1], 1);
        mbar_init(&bar_th, 1);
        mbar_init(&bar_b, 1);
        mbar_init(&bar_c, 1);
        mbar_init(&bar_yo, 1);
        mbar_init(&bar_s, 1);
        mbar_init(&bar_dh, 1);
        mbar_init(&bar_m2, 1);
        fence_mbar_init();
        s_abort = 0;
        s_issued[0] = s_issued[1] = -1;
        for (int i = 2; i < 7; ++i) s_issued[i] = 0;
        if (nchunks > 0) {
            issue_x(0);
            issue_sc(0);
            issue_th(0);
            issue_b(0);
            if constexpr (!kStateOnly) issue_c(0);
        }
        if (nchunks > 1) issue_sc(1);
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
    // the full pass of a cut sequence takes every start state from the workspace
    const bool from_ws = !kStateOnly && sa.nseg > 1;
    if (from_ws) {
        // segment 0's primed initial state; later segments assemble theirs below
        const float4* src = reinterpret_cast<const float4*>(
            sa.st + (u * sa.nseg + (kseg == 0 ? sa.nseg - 1 : 0)) * kSegStride + nrow * kP + 32 * wh);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float4 v = src[j];
            hreg[4 * j] = v.x; hreg[4 * j + 1] = v.y; hreg[4 * j + 2] = v.z; hreg[4 * j + 3] = v.w;
        }
    } else if (kseg == 0 && p.h0) {
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

    // Rotation mapping: warp = token segment (TPS consecutive tokens), lane = pair couple
    // (2 lane, 2 lane + 1) with partners (+ N/2). The cumulative angle of the couple, as stored
    // in the state (car) and reduced into [-pi, pi] once per chunk (car_r: Cody & Waite's
    // two-constant reduction, "Software Manual for the Elementary Functions", 1980), so that
    // the per-token angles stay small.
    const int jp = 2 * lane;
    float car[2], car_r[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        car[j] = (from_ws && kseg == 0) ? sa.st[(u * sa.nseg + sa.nseg - 1) * kSegStride + kN * kP + jp + j]
               : (!from_ws && kseg == 0 && p.phi0) ? p.phi0[u * kHalf + jp + j] : 0.f;
        car_r[j] = reduce_2pi(car[j]);
    }

    // ---- fold the stored previous token into the primed state ----
    if (!from_ws && kseg == 0 && p.h0 && L > 0) {
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
            const float b0 = p.Bbias ? p.Bbias[hh * R * kN + r * kN + i] : 0.f;
            const float b1 = p.Bbias ? p.Bbias[hh * R * kN + r * kN + i + kHalf] : 0.f;
            const float u0 = __bfloat162float(pB[r * kN + i]) * rs + b0;
            const float u1 = __bfloat162float(pB[r * kN + i + kHalf]) * rs + b1;
            s_fold[r * kN + i] = u0 * cs + u1 * sn;
            s_fold[r * kN + i + kHalf] = u1 * cs - u0 * sn;
        }
        __syncthreads();
        const int64_t s0 = bb * p.L * p.H + hh;
        const float f = (kRaw && (p.flags & 4u)) ? 0.f   // zero-order hold: no beta term
                        : (1.f - step_lam<kRaw>(p.lam[s0], p.flags)) * step_dt<kRaw>(p.dt[s0], dtb, p.flags);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            float acc = 0.f;
#pragma unroll
            for (int r = 0; r < R; ++r) acc = fmaf(s_fold[r * kN + nrow], s_foldx[r * kP + 32 * wh + j], acc);
            hreg[j] = fmaf(f, acc, hreg[j]);
        }
    }

    // ---- the state-only pass keeps segment 0's primed initial state for the full pass ----
    if constexpr (kStateOnly) {
        if (kseg == 0 && sa.save_init && !sa.out_h) {
            float* so = sa.st + (u * sa.nseg + sa.nseg - 1) * kSegStride;
            float4* dst = reinterpret_cast<float4*>(so + nrow * kP + 32 * wh);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                dst[j] = make_float4(hreg[4 * j], hreg[4 * j + 1], hreg[4 * j + 2], hreg[4 * j + 3]);
            if (warp == 0) {
                so[kN * kP + jp] = car[0];
                so[kN * kP + jp + 1] = car[1];
            }
        }
    }

    // ---- the state at the start of a later segment (full pass) ----
    // Segment 0's end state is in the true frame. Each later segment j < kseg adds its own
    // contribution dH_j, computed from zero in its own frame, after decaying the state by its
    // summed log-decay Lambda_j and rotating dH_j by the angle phi_j at its start:
    //     h <- e^{Lambda_j} h + R(-phi_j) dH_j,   phi_{j+1} = phi_j + (segment j's angle sum).
    // The states at segment boundaries are primed (they hold the next token's beta term, as at
    // every chunk boundary), so no previous token is folded here.
    if constexpr (!kStateOnly) {
        if (kseg > 0) {
            const float* sb = sa.st + u * sa.nseg * kSegStride;
            float* s_phis = reinterpret_cast<float*>(sm + Cfg::OH);   // [kseg][N/2], set-up only
            if (tid < kHalf) {
                float acc = sb[kN * kP + tid];
                s_phis[tid] = acc;
                for (int j = 1; j < kseg; ++j) {
                    acc += sb[j * kSegStride + kN * kP + tid];
                    s_phis[j * kHalf + tid] = acc;
                }
            }
            __syncthreads();
            const int prow = nrow ^ kHalf;   // the other half of this row's rotation pair
            for (int j = 1; j < kseg; ++j) {
                const float* sj = sb + j * kSegStride;
                const float e = expf(sj[kN * kP + kHalf]);
                float sn, cs;
                sincosf(s_phis[(j - 1) * kHalf + (nrow & (kHalf - 1))], &sn, &cs);
                // rows n < N/2: v_n cos + v_{n+N/2} sin; rows n >= N/2: v_n cos - v_{n-N/2} sin
                const float sg = nrow < kHalf ? sn : -sn;
                const float4* own = reinterpret_cast<const float4*>(sj + nrow * kP + 32 * wh);
                const float4* oth = reinterpret_cast<const float4*>(sj + prow * kP + 32 * wh);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const float4 a = own[q], b = oth[q];
                    hreg[4 * q] = fmaf(e, hreg[4 * q], fmaf(a.x, cs, b.x * sg));
                    hreg[4 * q + 1] = fmaf(e, hreg[4 * q + 1], fmaf(a.y, cs, b.y * sg));
                    hreg[4 * q + 2] = fmaf(e, hreg[4 * q + 2], fmaf(a.z, cs, b.z * sg));
                    hreg[4 * q + 3] = fmaf(e, hreg[4 * q + 3], fmaf(a.w, cs, b.w * sg));
                }
            }
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                car[j] = s_phis[(kseg - 1) * kHalf + jp + j];
                car_r[j] = reduce_2pi(car[j]);
            }
        }
    }

    const uint32_t aB = smem_u32(sm + Cfg::OB), aC = smem_u32(sm + Cfg::OC);
    const uint32_t aXP = smem_u32(sm + Cfg::XP), aH = smem_u32(sm + Cfg::OH);
    const uint32_t id_s = idesc_bf16(64, 64, false, false);   // S  = C . B^T
    const uint32_t id_yo = idesc_bf16(64, 64, false, true);   // Yo = C . H
    const uint32_t id_dh = idesc_bf16(128, 64, true, true);   // dH = B^T . X'
    const uint32_t id_yd = idesc_bf16(64, 64, false, true);   // Yd = P . X

    // y of chunk c from the Yd / Yo accumulators (TMEM): y = Yd + e^{cum_t} Yo
    auto epilogue = [&](int c) {
        float yd[16], yo[16];
        const uint32_t lanebase = (32u * q4) << 16;
        tmem_ld_16x32bx2_x16(tmem + lanebase + T_YD + 16u * wh, yd);
        tmem_ld_16x32bx2_x16(tmem + lanebase + T_YO + 16u * wh, yo);
        const int trow = 16 * q4 + (lane & 15);
        const int col0 = 16 * wh + ((lane >> 4) ? 32 : 0);
        const int t = trow / R, r = trow % R;
        const int c0 = (cb + c) * Q;
        const int T = (L - c0) < Q ? (L - c0) : Q;
        const float e = sf[(c & 1) * F_BLK + F_ECUM + t];
        tmem_wait_ld();
        if (t < T) {
            __nv_bfloat16* dst = yu + (c0 + t) * tokY + r * kP + col0;
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
    };

    // H0 (bf16) as the Yo operand: row nrow, columns [32 wh, 32 wh + 32)
    auto store_h0 = [&]() {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint4 v;
            v.x = pack_bf16(hreg[8 * i + 0], hreg[8 * i + 1]);
            v.y = pack_bf16(hreg[8 * i + 2], hreg[8 * i + 3]);
            v.z = pack_bf16(hreg[8 * i + 4], hreg[8 * i + 5]);
            v.w = pack_bf16(hreg[8 * i + 6], hreg[8 * i + 7]);
            *reinterpret_cast<uint4*>(sm + Cfg::OH + swz128(nrow, 32 * wh + 8 * i)) = v;
        }
    };

    // One couple of rotation pairs (jp, jp + 1) of one operand row: byte offset o in the two
    // 64-column slabs of src (raw, bf16) and dst (rotated, bf16); bias at [jp] and [jp + 64].
    auto rotate_couple = [&](const uint8_t* src, uint8_t* dst, uint32_t o, float rs,
                             const float* bias, float2 c, float2 s) {
        const float2 r2 = make_float2(rs, rs);
        const float2 u0 = __ffma2_rn(bf2_to_f2(*reinterpret_cast<const uint32_t*>(src + o)), r2,
                                     *reinterpret_cast<const float2*>(bias));
        const float2 u1 = __ffma2_rn(bf2_to_f2(*reinterpret_cast<const uint32_t*>(src + 8192 + o)),
                                     r2, *reinterpret_cast<const float2*>(bias + kHalf));
        *reinterpret_cast<uint32_t*>(dst + o) = f2_to_bf2(__ffma2_rn(u0, c, __fmul2_rn(u1, s)));
        *reinterpret_cast<uint32_t*>(dst + 8192 + o) =
            f2_to_bf2(__ffma2_rn(u1, c, __fmul2_rn(make_float2(-u0.x, -u0.y), s)));
    };

    // Angles and rotation of chunk c (I1): the cumulative angle of every token, then B and C
    // (B only in the state-only pass) normalised, biased and rotated into their operand tiles.
    auto rotate = [&](const float* blk, uint32_t par) {
        // Angle increments dt_t theta_t of the segment's tokens, their sum per pair, and the
        // segment totals exchanged through shared memory: each lane then walks its own
        // tokens from carry + the earlier segments' totals.
        float inc[TPS][2];
        float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
        for (int k = 0; k < TPS; ++k) {
            const int t = warp * TPS + k;
            const uint32_t th = *reinterpret_cast<const uint32_t*>(sm + Cfg::TH + swz128(t, jp));
            const float dd = blk[F_DT + t];  // 0 past the sequence end: no rotation there
            inc[k][0] = dd * __uint_as_float(th << 16);
            inc[k][1] = dd * __uint_as_float(th & 0xFFFF0000u);
            sum0 += inc[k][0];
            sum1 += inc[k][1];
        }
        s_seg[warp * 32 + lane] = make_float2(sum0, sum1);
        __syncthreads();
        float a0 = car_r[0], a1 = car_r[1], tot0 = 0.f, tot1 = 0.f;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const float2 v = s_seg[k * 32 + lane];
            if (k < warp) { a0 += v.x; a1 += v.y; }
            tot0 += v.x;
            tot1 += v.y;
        }
        car[0] += tot0;
        car[1] += tot1;
        car_r[0] = reduce_2pi(car_r[0] + tot0);
        car_r[1] = reduce_2pi(car_r[1] + tot1);
        // Each token's angle, then its cos and sin: before the raw B and C have landed when
        // they fit in registers (two tokens or fewer per warp), else token by token below.
        constexpr bool kEarly = TPS <= 2;
        float2 cse[kEarly ? TPS : 1], sne[kEarly ? TPS : 1];
        if constexpr (kEarly) {
#pragma unroll
            for (int k = 0; k < TPS; ++k) {
                a0 += inc[k][0];
                a1 += inc[k][1];
                __sincosf(a0, &sne[k].x, &cse[k].x);
                __sincosf(a1, &sne[k].y, &cse[k].y);
            }
        }
        if (!mbar_wait(&bar_b, par)) s_abort = 1;   // raw B and the RMS scales
        if constexpr (!kStateOnly) {
            if (!mbar_wait(&bar_c, par)) s_abort = 1;   // raw C
        }
        // Every rank's B (and C) row at the couple: u = rs raw + bias on both halves of each
        // pair, (u0, u1) -> (u0 c + u1 s, u1 c - u0 s), all in fp32 with one rounding to bf16.
#pragma unroll
        for (int k = 0; k < TPS; ++k) {
            float2 cs, sn;
            if constexpr (kEarly) {
                cs = cse[k];
                sn = sne[k];
            } else {
                a0 += inc[k][0];
                a1 += inc[k][1];
                __sincosf(a0, &sn.x, &cs.x);
                __sincosf(a1, &sn.y, &cs.y);
            }
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const int row = (warp * TPS + k) * R + r;
                const uint32_t o = swz128(row, jp);
                const float2 rsv = rsu ? s_rs[row] : make_float2(1.f, 1.f);
                rotate_couple(sm + Cfg::RB, sm + Cfg::OB, o, rsv.x, s_biasB + r * kN + jp, cs, sn);
                if constexpr (!kStateOnly)
                    rotate_couple(sm + Cfg::OC, sm + Cfg::OC, o, rsv.y, s_biasC + r * kN + jp, cs, sn);
            }
        }
    };

    // X' = diag(dw) X of chunk c into the XP buffer (whose previous readers have finished)
    auto xprime = [&](int c, const float* blk) {
        const int st = c & 1;
        uint8_t* sX = sm + (st ? Cfg::X1 : Cfg::X0);
        if (!mbar_wait(&bar_x[st], (c >> 1) & 1)) s_abort = 1;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int e = tid + i * kTcThreads;
            const int row = e >> 3, ch = e & 7;
            const float dw = blk[F_DW + row / R];
            const float2 dw2 = make_float2(dw, dw);
            const uint32_t o = static_cast<uint32_t>(row) * 128u + (static_cast<uint32_t>(ch) << 4);
            uint4 v = *reinterpret_cast<const uint4*>(sX + o);   // x dw in fp32, one rounding
            v.x = f2_to_bf2(__fmul2_rn(bf2_to_f2(v.x), dw2));
            v.y = f2_to_bf2(__fmul2_rn(bf2_to_f2(v.y), dw2));
            v.z = f2_to_bf2(__fmul2_rn(bf2_to_f2(v.z), dw2));
            v.w = f2_to_bf2(__fmul2_rn(bf2_to_f2(v.w), dw2));
            *reinterpret_cast<uint4*>(sm + Cfg::XP + o) = v;
        }
    };

    if constexpr (kStateOnly) {
        if constexpr (kRaw) {
            if (nchunks > 0) {
                if (!mbar_wait(&bar_sc[0], 0)) s_abort = 1;
                raw_box(0);
                __syncthreads();
            }
        }
        if (nchunks > 0 && warp == 3) scalars(0);
        __syncthreads();   // also: the fold's scratch in the H0 buffer has been read
        for (int c = 0; c < nchunks && !s_abort; ++c) {
            const int st = c & 1;
            const uint32_t par = static_cast<uint32_t>(c & 1);
            const float* blk = sf + st * F_BLK;
            // ======== I1: angles and rotation of B; X(c+1) (its buffer was last read by X'(c-1));
            // the X' operand ========
            if constexpr (kRaw) {
                if (c + 1 < nchunks) {   // the next chunk's raw scalars, for scalars(c+1) in I2, while
                                         // theta(c) lands
                    if (!mbar_wait(&bar_sc[(c + 1) & 1], ((c + 1) >> 1) & 1)) s_abort = 1;
                    raw_box(c + 1);
                }
            }
            if (sa.chunk_h) {
                // the primed state before this chunk, scaled by its first token's decay, and the
                // angle before it, for the backward's per-chunk products
                const float e0 = blk[F_ECUM];
                uint8_t* dst = sa.chunk_h + (u * nchunks + c) * 16384;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    uint4 v;
                    v.x = pack_bf16(e0 * hreg[8 * i + 0], e0 * hreg[8 * i + 1]);
                    v.y = pack_bf16(e0 * hreg[8 * i + 2], e0 * hreg[8 * i + 3]);
                    v.z = pack_bf16(e0 * hreg[8 * i + 4], e0 * hreg[8 * i + 5]);
                    v.w = pack_bf16(e0 * hreg[8 * i + 6], e0 * hreg[8 * i + 7]);
                    *reinterpret_cast<uint4*>(dst + swz128(nrow, 32 * wh + 8 * i)) = v;
                }
                if (warp == 0)
                    *reinterpret_cast<float2*>(sa.chunk_phi + (u * nchunks + c) * kHalf + jp) =
                        make_float2(car[0], car[1]);
            }
            if (!mbar_wait(&bar_th, par)) s_abort = 1;   // theta of this chunk
            rotate(blk, par);
            if (warp == kIssueWarp) {
                if (elect_one() && c + 1 < nchunks) issue_x(c + 1);
                __syncwarp();
            }
            xprime(c, blk);   // XP was last read by dH(c-1), waited for by every thread
            fence_proxy_async();
            fence_before_sync();
            __syncthreads();
            fence_after_sync();
            if (s_abort) break;
            // ======== I2: dH on the tensor cores, the next chunk's scalars meanwhile, then
            // H1 = e^{cum_end} H0 + dH ========
            if (warp == kIssueWarp) {
                if (elect_one()) {
                    if (c + 1 < nchunks) {
                        issue_th(c + 1);
                        issue_b(c + 1);
                    }
                    if (c + 2 < nchunks) issue_sc(c + 2);
                    constexpr uint32_t hi = desc_hi_sw128(1024);
                    const uint32_t loBt = desc_lo(aB, 8192), loXP = desc_lo(aXP, 8192);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        mma_bf16(tmem + T_DH, desc_pack(loBt + (mnmajor_off(k) >> 4), hi),
                                 desc_pack(loXP + (mnmajor_off(k) >> 4), hi), id_dh, k > 0);
                    mma_commit(smem_u32(&bar_dh));
                    s_issued[5] = c + 1;
                }
                __syncwarp();
            }
            if (warp == 3 && c + 1 < nchunks) scalars(c + 1);
            {
                if (!mbar_wait(&bar_dh, par)) s_abort = 1;
                fence_after_sync();
                const float eend = blk[F_MISC];
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
            // the next chunk's scalars are published; dH has been read out of TMEM
            fence_before_sync();
            __syncthreads();
            fence_after_sync();
        }
    } else {
        if constexpr (kRaw) {
            if (nchunks > 0) {
                if (!mbar_wait(&bar_sc[0], 0)) s_abort = 1;
                raw_box(0);
                __syncthreads();
            }
        }
        if (nchunks > 0 && warp == 3) scalars(0);
        __syncthreads();   // also: the fold's scratch in the H0 buffer has been read
        store_h0();

        for (int c = 0; c < nchunks && !s_abort; ++c) {
            const int st = c & 1;
            const uint32_t par = static_cast<uint32_t>(c & 1);
            const float* blk = sf + st * F_BLK;

            // ======== I1: rotation(c); then epilogue(c-1), the H0 and X' operands ========
            if constexpr (kRaw) {
                if (c + 1 < nchunks) {   // the next chunk's raw scalars, for scalars(c+1) in I2, while
                                         // theta(c) lands
                    if (!mbar_wait(&bar_sc[(c + 1) & 1], ((c + 1) >> 1) & 1)) s_abort = 1;
                    raw_box(c + 1);
                }
            }
            if (!mbar_wait(&bar_th, par)) s_abort = 1;   // theta of this chunk
            rotate(blk, par);
            // Yd(c-1) done: its X buffer takes X(c+1), and y(c-1) can be written
            if (warp == kIssueWarp) {
                if (elect_one()) {
                    if (c > 0 && !mbar_wait(&bar_m2, (c - 1) & 1)) s_abort = 1;
                    if (c + 1 < nchunks) issue_x(c + 1);
                }
                __syncwarp();
            }
            if (c > 0) {
                (void)mbar_wait(&bar_m2, (c - 1) & 1);
                fence_after_sync();
                epilogue(c - 1);
            }
            // X' = diag(dw) X (the XP buffer held P(c-1), read by Yd(c-1), which has finished)
            xprime(c, blk);
            fence_proxy_async();
            fence_before_sync();
            __syncthreads();
            fence_after_sync();
            if (s_abort) break;

            // ======== I2: Yo, S, dH on the tensor cores; P = S o M and H1 = e^{cum_end} H0 + dH
            // as their accumulators land; the next chunk's scalars meanwhile ========
            if (warp == kIssueWarp) {
                if (elect_one()) {
                    // theta and raw B of chunk c+1 (their buffers were read by the rotation), the
                    // scalar boxes of chunk c+2 (chunk c's slot was read by scalars(c))
                    if (c + 1 < nchunks) {
                        if (!(blockIdx.x == 0 && c + 1 == p.test_skip_theta)) issue_th(c + 1);
                        issue_b(c + 1);
                    }
                    if (c + 2 < nchunks) issue_sc(c + 2);
                    constexpr uint32_t hi = desc_hi_sw128(1024);
                    const uint32_t loC = desc_lo(aC, 16), loB = desc_lo(aB, 16);
                    const uint32_t loBt = desc_lo(aB, 8192), loXP = desc_lo(aXP, 8192);
                    const uint32_t loH = desc_lo(aH, 16384);
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        mma_bf16(tmem + T_YO, desc_pack(loC + (kmajor_off(k, 8192) >> 4), hi),
                                 desc_pack(loH + (mnmajor_off(k) >> 4), hi), id_yo, k > 0);
                    mma_commit(smem_u32(&bar_yo));
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        mma_bf16(tmem + T_S, desc_pack(loC + (kmajor_off(k, 8192) >> 4), hi),
                                 desc_pack(loB + (kmajor_off(k, 8192) >> 4), hi), id_s, k > 0);
                    mma_commit(smem_u32(&bar_s));
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        mma_bf16(tmem + T_DH, desc_pack(loBt + (mnmajor_off(k) >> 4), hi),
                                 desc_pack(loXP + (mnmajor_off(k) >> 4), hi), id_dh, k > 0);
                    mma_commit(smem_u32(&bar_dh));
                    s_issued[5] = c + 1;
                    // Yo and S were the readers of Cbar: fetch the next chunk's raw C in its place
                    if (c + 1 < nchunks) {
                        if (!mbar_wait(&bar_s, par)) s_abort = 1;
                        issue_c(c + 1);
                    }
                }
                __syncwarp();
            }
            if (warp == 3 && c + 1 < nchunks) scalars(c + 1);
            {
                const int trow = 16 * q4 + (lane & 15);   // row block q4
                const int qc = wh + ((lane >> 4) ? 2 : 0);  // column block of this half-warp
                const int col0 = 16 * qc;
                const int t = trow / R;
                constexpr int NT = 16 / R;                  // tokens covered by the 16 columns
                const int s0 = col0 / R;
                float m[NT];
                if (qc < q4) {          // strictly below the diagonal block: factored decay
                    const float er = blk[F_EROW + t];
#pragma unroll
                    for (int i = 0; i < NT; i += 2) {
                        const float2 e2 = *reinterpret_cast<const float2*>(blk + F_ECOL + (q4 - 1) * 64 + s0 + i);
                        m[i] = er * e2.x;
                        m[i + 1] = er * e2.y;
                    }
                } else if (qc == q4) {  // diagonal block: decay, trapezoid weight and gamma
                    const float cum_t = blk[F_CUM + t], gam_t = blk[F_GAM + t];
#pragma unroll
                    for (int i = 0; i < NT; i += 2) {
                        const float2 a2 = *reinterpret_cast<const float2*>(blk + F_CUM + s0 + i);
                        const float2 w2 = *reinterpret_cast<const float2*>(blk + F_W + s0 + i);
                        const int sa = s0 + i;
                        m[i] = (sa < t) ? ex2_approx(fminf(cum_t - a2.x, 0.f)) * w2.x : ((sa == t) ? gam_t : 0.f);
                        m[i + 1] = (sa + 1 < t) ? ex2_approx(fminf(cum_t - a2.y, 0.f)) * w2.y
                                                : ((sa + 1 == t) ? gam_t : 0.f);
                    }
                } else {                // above the diagonal: zero
#pragma unroll
                    for (int i = 0; i < NT; ++i) m[i] = 0.f;
                }
                if (!mbar_wait(&bar_s, par)) s_abort = 1;
                fence_after_sync();
                float sv[16];
                tmem_ld_16x32bx2_x16(tmem + ((32u * q4) << 16) + T_S + 16u * wh, sv);
                tmem_wait_ld();
                uint32_t pw[8];
#pragma unroll
                for (int j = 0; j < 16; j += 2)
                    pw[j / 2] = pack_bf16(sv[j] * m[j / R], sv[j + 1] * m[(j + 1) / R]);
                // dH has read X': P takes its buffer
                if (!mbar_wait(&bar_dh, par)) s_abort = 1;
                fence_after_sync();
                *reinterpret_cast<uint4*>(sm + Cfg::XP + swz128(trow, col0)) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
                *reinterpret_cast<uint4*>(sm + Cfg::XP + swz128(trow, col0 + 8)) = make_uint4(pw[4], pw[5], pw[6], pw[7]);
            }
            {
                const float eend = blk[F_MISC];
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
            // Yo(c) has read H0: the next chunk's H0 operand
            if (!mbar_wait(&bar_yo, par)) s_abort = 1;
            store_h0();

            fence_proxy_async();
            fence_before_sync();
            __syncthreads();
            fence_after_sync();
            if (s_abort) break;

            // ======== I4: Yd = P X (waited for in the next chunk's I1) ========
            if (warp == kIssueWarp) {
                if (elect_one()) {
                    constexpr uint32_t hi = desc_hi_sw128(1024);
                    const uint32_t loP = desc_lo(aXP, 16);
                    const uint32_t loX = desc_lo(smem_u32(sm + (st ? Cfg::X1 : Cfg::X0)), 8192);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        mma_bf16(tmem + T_YD, desc_pack(loP + (kmajor_off(k, 8192) >> 4), hi),
                                 desc_pack(loX + (mnmajor_off(k) >> 4), hi), id_yd, k > 0);
                    mma_commit(smem_u32(&bar_m2));
                    s_issued[6] = c + 1;
                }
                __syncwarp();
            }
        }
        // ---- epilogue of the last chunk ----
        if (nchunks > 0 && !s_abort) {
            if (tid == 0 && !mbar_wait(&bar_m2, (nchunks - 1) & 1)) s_abort = 1;
            fence_before_sync();
            __syncthreads();
            fence_after_sync();
            if (!s_abort) {
                (void)mbar_try_wait(smem_u32(&bar_m2), (nchunks - 1) & 1);
                epilogue(nchunks - 1);
            }
        }
    }

    // ---------------- final state ----------------
    __syncthreads();
    if (!s_abort && kStateOnly) {
        // this segment's end state: h, the angle sum (absolute for segment 0), the summed
        // log-decay; into the workspace for the full pass, or to the caller (m3_scan_state)
        float* so = sa.out_h ? sa.out_h + u * kN * kP : sa.st + (u * sa.nseg + kseg) * kSegStride;
        float* sphi = sa.out_h ? sa.out_phi + u * kHalf : so + kN * kP;
        float* slam = sa.out_h ? sa.out_lam + u : so + kN * kP + kHalf;
        float4* dst = reinterpret_cast<float4*>(so + nrow * kP + 32 * wh);
#pragma unroll
        for (int j = 0; j < 8; ++j)
            dst[j] = make_float4(hreg[4 * j], hreg[4 * j + 1], hreg[4 * j + 2], hreg[4 * j + 3]);
        if (warp == 0) {
            sphi[jp] = car[0];
            sphi[jp + 1] = car[1];
        }
        if (warp == 3 && lane == 0) *slam = lam_acc;
    } else if (!s_abort) {
        // the sequence's final state, written by its last segment
        if (kseg == sa.nseg - 1) {
            if (p.h1) {
                float4* dst = reinterpret_cast<float4*>(p.h1 + (u * kN + nrow) * kP + 32 * wh);
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    dst[j] = make_float4(hreg[4 * j], hreg[4 * j + 1], hreg[4 * j + 2], hreg[4 * j + 3]);
            }
            if (p.phi1 && warp == 0) {
                p.phi1[u * kHalf + jp] = car[0];
                p.phi1[u * kHalf + jp + 1] = car[1];
            }
            if (L > 0) {
                if (p.prevB1) {
                    __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.prevB1) + u * R * kN;
                    const __nv_bfloat16* src = Bu + (L - 1) * tokB;
                    for (int e = tid; e < R * kN; e += kTcThreads) dst[e] = src[e];
                }
                if (p.prevx1) {
                    __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.prevx1) + u * R * kP;
                    const __nv_bfloat16* src = xu + (L - 1) * tokY;
                    for (int e = tid; e < R * kP; e += kTcThreads) dst[e] = src[e];
                }
            }
        }
    } else if (tid == 0) {
        if (p.status) atomicExch(p.status, 1);
        // A wait gave up: let this CTA's own TMA copies and MMAs finish (bounded) before the
        // shared memory and TMEM they target are released.
        constexpr long long kDrain = 200000000LL;
        for (int k = s_issued[0] - 1; k <= s_issued[0]; ++k)
            if (k >= 0) (void)mbar_wait(&bar_x[k & 1], (k >> 1) & 1, kDrain);
        for (int k = s_issued[1] - 1; k <= s_issued[1]; ++k)
            if (k >= 0) (void)mbar_wait(&bar_sc[k & 1], (k >> 1) & 1, kDrain);
        if (s_issued[2] > 0) (void)mbar_wait(&bar_th, (s_issued[2] - 1) & 1, kDrain);
        if (s_issued[3] > 0) (void)mbar_wait(&bar_b, (s_issued[3] - 1) & 1, kDrain);
        if (s_issued[4] > 0) (void)mbar_wait(&bar_c, (s_issued[4] - 1) & 1, kDrain);
        if (s_issued[5] > 0) {
            if constexpr (!kStateOnly) {
                (void)mbar_wait(&bar_yo, (s_issued[5] - 1) & 1, kDrain);
                (void)mbar_wait(&bar_s, (s_issued[5] - 1) & 1, kDrain);
            }
            (void)mbar_wait(&bar_dh, (s_issued[5] - 1) & 1, kDrain);
        }
        if (s_issued[6] > 0) (void)mbar_wait(&bar_m2, (s_issued[6] - 1) & 1, kDrain);
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

bool encode(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base,
            const cuuint64_t* dims, const cuuint64_t* strides, const cuuint32_t* box,
            CUtensorMapSwizzle swz) {
    auto enc = get_encode();
    if (!enc) return false;
    const cuuint32_t es[5] = {1, 1, 1, 1, 1};
    return enc(m, dt, static_cast<cuuint32_t>(rank), const_cast<void*>(base), dims, strides, box,
               es, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool tc_scan_supported(const ScanParams& p, bool bf16) {
    // 32-bit element offsets inside one sequence: L * G * R * N and L * H * R * P < 2^31
    const int64_t lim = 0x7fffffffLL;
    return bf16 && p.N == kN && p.P == kP && p.Q * p.R == 64 &&
           (p.R == 1 || p.R == 2 || p.R == 4 || p.R == 8) && p.H % 4 == 0 &&
           p.L * p.G * p.R * kN < lim && p.L * p.H * p.R * kP < lim && p.b <= lim;
}

namespace {

// Segments per sequence. When the (batch, head) units alone would leave SMs idle, each
// sequence is cut so that units x segments fills every SM twice (two CTAs per SM), keeping at
// least kMinSegChunks chunks per segment and at most kMaxSeg segments, and no more segments
// than seg_bytes of workspace can hold the end states of.
constexpr int64_t kMinSegChunks = 8, kMaxSeg = 16;
SegArgs seg_plan(const ScanParams& p, size_t seg_bytes = ~size_t(0)) {
    const int64_t Q = 64 / (p.R > 0 ? p.R : 1);
    const int64_t nch = (p.L + Q - 1) / Q;
    const int64_t units = p.b * p.H;
    SegArgs sa{static_cast<int>(nch), 1, nullptr, nullptr, nullptr, nullptr};
    if (units <= 0 || nch == 0) return sa;
    int64_t S = 2 * device_sm_count() / units;
    S = std::min(S, nch / kMinSegChunks);
    S = std::min(S, kMaxSeg);
    const size_t per_seg = static_cast<size_t>(units) * kSegStride * sizeof(float);
    while (S >= 2 && static_cast<size_t>(S) * per_seg > seg_bytes) --S;   // nseg slots per unit
    if (S < 2) return sa;
    sa.seg_chunks = static_cast<int>((nch + S - 1) / S);
    sa.nseg = static_cast<int>((nch + sa.seg_chunks - 1) / sa.seg_chunks);
    return sa;
}

size_t rs_bytes(const ScanParams& p) {
    const int64_t Q = 64 / (p.R > 0 ? p.R : 1);
    const int64_t Lpad = (p.L + Q - 1) / Q * Q;
    const size_t n = p.bc_norm ? static_cast<size_t>(p.b * Lpad * p.G * p.R) * sizeof(float2) : 0;
    return (n + 255) / 256 * 256;
}

}  // namespace

cudaError_t launch_rms_scales(const ScanParams& p, int64_t Q, float2* out, cudaStream_t s) {
    const int64_t rows = p.b * p.L * p.G * p.R;
    if (rows == 0) return cudaSuccess;
    const int64_t Lpad = (p.L + Q - 1) / Q * Q;
    const int64_t all = rows + p.b * p.G * (Lpad - p.L) * p.R;   // padded rows get zero scales
    rms_scale_kernel<<<static_cast<unsigned>((all + 7) / 8), 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(p.B), static_cast<const __nv_bfloat16*>(p.C), rows,
        p.L, p.G, p.R, Lpad, p.eps, out);
    return cudaGetLastError();
}

size_t tc_scan_workspace_bytes(const ScanParams& p) {
    const SegArgs sa = seg_plan(p);
    const size_t seg = sa.nseg > 1 ? static_cast<size_t>(p.b * p.H) * sa.nseg * kSegStride * sizeof(float) : 0;
    return rs_bytes(p) + seg;
}

size_t tc_scan_workspace_min_bytes(const ScanParams& p) { return rs_bytes(p); }

template <int R, bool kRaw>
static cudaError_t launch_tc_t(const ScanParams& p, float2* rs, const SegArgs& sa, cudaStream_t s,
                               bool state_only = false) {
    constexpr int Q = 64 / R;
    TcMaps maps;
    const cuuint64_t H = p.H, Lq = p.L, b = p.b;
    {   // x [b][L][H][R][P], box (P, R, 1, Q, 1)
        const cuuint64_t dims[5] = {kP, static_cast<cuuint64_t>(R), H, Lq, b};
        const cuuint64_t str[4] = {kP * 2, R * kP * 2, H * R * kP * 2, Lq * H * R * kP * 2};
        const cuuint32_t box[5] = {kP, static_cast<cuuint32_t>(R), 1, Q, 1};
        if (!encode(&maps.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, p.x, dims, str, box,
                    CU_TENSOR_MAP_SWIZZLE_128B)) return cudaErrorInvalidValue;
    }
    {   // theta [b][L][H][N/2], box (64, 1, Q, 1)
        const cuuint64_t dims[4] = {kHalf, H, Lq, b};
        const cuuint64_t str[3] = {kHalf * 2, H * kHalf * 2, Lq * H * kHalf * 2};
        const cuuint32_t box[4] = {kHalf, 1, Q, 1};
        if (!encode(&maps.theta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, p.theta, dims, str, box,
                    CU_TENSOR_MAP_SWIZZLE_128B)) return cudaErrorInvalidValue;
    }
    {   // B, C [b][L][G][R][N], box (64 columns, R, 1, Q, 1): one 64-column slab per load
        const cuuint64_t Gq = p.G;
        const cuuint64_t dims[5] = {kN, static_cast<cuuint64_t>(R), Gq, Lq, b};
        const cuuint64_t str[4] = {kN * 2, R * kN * 2, Gq * R * kN * 2, Lq * Gq * R * kN * 2};
        const cuuint32_t box[5] = {kHalf, static_cast<cuuint32_t>(R), 1, Q, 1};
        if (!encode(&maps.B, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, p.B, dims, str, box,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
            !encode(&maps.C, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, p.C, dims, str, box,
                    CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
    }
    {   // dt, A, lam [b][L][H] fp32, box (4 heads, Q + 1 tokens, 1)
        const cuuint64_t dims[3] = {H, Lq, b};
        const cuuint64_t str[2] = {H * 4, Lq * H * 4};
        const cuuint32_t box[3] = {4, Q + 1, 1};
        if (!encode(&maps.dt, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, p.dt, dims, str, box,
                    CU_TENSOR_MAP_SWIZZLE_NONE) ||
            !encode(&maps.A, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, p.A, dims, str, box,
                    CU_TENSOR_MAP_SWIZZLE_NONE) ||
            !encode(&maps.lam, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, p.lam, dims, str, box,
                    CU_TENSOR_MAP_SWIZZLE_NONE))
            return cudaErrorInvalidValue;
    }
    if (rs) {
        cudaError_t e = launch_rms_scales(p, Q, rs, s);
        if (e != cudaSuccess) return e;
    }
    const uint32_t smem = tc_smem_bytes<R>();
    const int64_t units = p.b * p.H;
    // the first scan kernel after the scales' kernel may start while that one finishes (it
    // waits for it only before its first load of the scales)
    bool first = rs != nullptr;
    auto launch = [&](auto kern, int64_t grid) -> cudaError_t {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        if (first) {
            first = false;
            return launch_after_rms(kern, static_cast<unsigned>(grid), kTcThreads, smem, s, p,
                                    maps, static_cast<const float2*>(rs), sa);
        }
        kern<<<static_cast<unsigned>(grid), kTcThreads, smem, s>>>(p, maps, rs, sa);
        return cudaGetLastError();
    };
    if (state_only)   // m3_scan_state: every segment's end state
        return launch(scan_tc_kernel<R, true, kRaw>, units * (sa.out_h ? 1 : sa.nseg));
    if (sa.nseg > 1) {   // every segment's end state but the last's
        cudaError_t e = launch(scan_tc_kernel<R, true, kRaw>, units * (sa.nseg - 1));
        if (e != cudaSuccess) return e;
    }
    return launch(scan_tc_kernel<R, false, kRaw>, units * sa.nseg);
}

bool encode_tmap(void* map, bool bf16, int rank, const void* base, const uint64_t* dims,
                 const uint64_t* strides, const uint32_t* box, bool swizzle128) {
    cuuint64_t d[5], st[4];
    cuuint32_t bx[5];
    for (int i = 0; i < rank; ++i) {
        d[i] = dims[i];
        bx[i] = box[i];
        if (i + 1 < rank) st[i] = strides[i];
    }
    return encode(static_cast<CUtensorMap*>(map),
                  bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, rank,
                  base, d, st, bx, swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE);
}

cudaError_t launch_bwd_states_tc(const ScanParams& p_in, float2* rs, uint8_t* chunk_h,
                                 float* chunk_phi, float* hfin, float* phifin, float* lamfin,
                                 cudaStream_t s) {
    if (p_in.b * p_in.H == 0) return cudaErrorInvalidValue;
    ScanParams p = p_in;
    p.Q = 64 / p.R;
    SegArgs sa;
    sa.seg_chunks = static_cast<int>((p.L + p.Q - 1) / p.Q);
    sa.nseg = 1;
    sa.out_h = hfin;
    sa.out_phi = phifin;
    sa.out_lam = lamfin;
    sa.save_init = false;
    sa.chunk_h = chunk_h;
    sa.chunk_phi = chunk_phi;
    const bool raw = p.flags != 0;
    switch (p.R) {
        case 1: return raw ? launch_tc_t<1, true>(p, rs, sa, s, true) : launch_tc_t<1, false>(p, rs, sa, s, true);
        case 2: return raw ? launch_tc_t<2, true>(p, rs, sa, s, true) : launch_tc_t<2, false>(p, rs, sa, s, true);
        case 4: return raw ? launch_tc_t<4, true>(p, rs, sa, s, true) : launch_tc_t<4, false>(p, rs, sa, s, true);
        case 8: return raw ? launch_tc_t<8, true>(p, rs, sa, s, true) : launch_tc_t<8, false>(p, rs, sa, s, true);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_scan_state_tc(const ScanParams& p, void* ws_body, size_t body_bytes,
                                 float* out_h, float* out_phi, float* out_lam, cudaStream_t s) {
    if (p.b * p.H == 0) return cudaSuccess;
    float2* rs = p.bc_norm ? static_cast<float2*>(ws_body) : nullptr;
    if (body_bytes < rs_bytes(p)) return cudaErrorInvalidValue;
    // few long sequences: the sequence-parallel form, every segment's end state into the
    // workspace, then their combination; else one segment straight into out
    SegArgs sa = seg_plan(p, body_bytes - rs_bytes(p));
    if (sa.nseg > 1) {
        sa.st = reinterpret_cast<float*>(static_cast<char*>(ws_body) + rs_bytes(p));
        sa.save_init = false;
    } else {
        sa.out_h = out_h;
        sa.out_phi = out_phi;
        sa.out_lam = out_lam;
    }
    const bool raw = p.flags != 0;
    cudaError_t e;
    switch (p.R) {
        case 1: e = raw ? launch_tc_t<1, true>(p, rs, sa, s, true) : launch_tc_t<1, false>(p, rs, sa, s, true); break;
        case 2: e = raw ? launch_tc_t<2, true>(p, rs, sa, s, true) : launch_tc_t<2, false>(p, rs, sa, s, true); break;
        case 4: e = raw ? launch_tc_t<4, true>(p, rs, sa, s, true) : launch_tc_t<4, false>(p, rs, sa, s, true); break;
        case 8: e = raw ? launch_tc_t<8, true>(p, rs, sa, s, true) : launch_tc_t<8, false>(p, rs, sa, s, true); break;
        default: return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess || sa.nseg <= 1) return e;
    const int64_t S = sa.nseg;
    const SegSrc src{sa.st, kSegStride, S * kSegStride, sa.st + kN * kP, kSegStride, S * kSegStride,
                     sa.st + kN * kP + kHalf, kSegStride, S * kSegStride};
    return launch_state_combine(p.b * p.H, kN, kP, sa.nseg, src, out_h, out_phi, out_lam, s);
}

cudaError_t launch_scan_tc(const ScanParams& p_in, void* ws_body, size_t body_bytes, cudaStream_t s) {
    if (p_in.b * p_in.H == 0) return cudaSuccess;
    ScanParams p = p_in;
    if (const char* e = std::getenv("M3_TEST_SKIP_THETA_LOAD")) p.test_skip_theta = std::atoi(e);
    // workspace body: the RMS scales, then the segments' end states
    float2* rs = p.bc_norm ? static_cast<float2*>(ws_body) : nullptr;
    if (body_bytes < rs_bytes(p)) return cudaErrorInvalidValue;
    SegArgs sa = seg_plan(p, body_bytes - rs_bytes(p));
    if (sa.nseg > 1) sa.st = reinterpret_cast<float*>(static_cast<char*>(ws_body) + rs_bytes(p));
    const bool raw = p.flags != 0;
    switch (p.R) {
        case 1: return raw ? launch_tc_t<1, true>(p, rs, sa, s) : launch_tc_t<1, false>(p, rs, sa, s);
        case 2: return raw ? launch_tc_t<2, true>(p, rs, sa, s) : launch_tc_t<2, false>(p, rs, sa, s);
        case 4: return raw ? launch_tc_t<4, true>(p, rs, sa, s) : launch_tc_t<4, false>(p, rs, sa, s);
        case 8: return raw ? launch_tc_t<8, true>(p, rs, sa, s) : launch_tc_t<8, false>(p, rs, sa, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace m3
