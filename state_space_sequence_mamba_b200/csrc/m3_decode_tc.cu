// One-token decode step with the rank-2R state update and the readout on the tensor cores.
//
// One iteration of the exponential-trapezoidal recurrence in the rotated frame per (batch,
// head) unit ("Mamba-3: Improved Sequence Modeling using State Space Principles", Sec. 3.1.1
// Prop. 1, Sec. 3.2.2 Prop. 4, Sec. 3.3 for MIMO, Appendix C):
//     h'  = alpha h + sum_r ( beta Bbar_prev[r] x_prev[r]^T + gamma Bbar[r] x[r]^T )
//     y[r] = Cbar[r]^T h'
// The sum over ranks is a K = 2R matrix product, U = [beta Bbar_prev | gamma Bbar] [x_prev ; x],
// and the readout a K = N one: the MIMO rank costs tensor-core FLOPs, which are otherwise idle
// here, instead of CUDA-core FMAs. Per unit:
//   1. rotation and scaling of B, B_prev and C (CUDA cores) into bf16 operand tiles;
//   2. U = A_U B_U on the tensor cores (M128 N64 K16, fp32 accumulator in TMEM);
//   3. h' = alpha h + U in fp32 on the CUDA cores, one FMA per element, on the fp32 state tile
//      that TMA brought in, written back in place. The tile uses the 128-byte swizzle with
//      32-byte atoms (32-byte chunk c of row r at c ^ (r mod 4)), the layout the tensor core
//      takes for an MN-major 32-bit operand. While the readout MMA runs, all threads copy the
//      tile to HBM with coalesced 16-byte stores (a swizzled TMA store drains too slowly to
//      free the slot in time);
//   4. y^T = h'^T Cbar^T on the tensor cores (kind::tf32, M64 N8 K128), reading that fp32 tile
//      directly as an MN-major operand.
// CTAs are persistent (two per SM) and walk a strided list of units with a two-deep ring of
// state tiles and small inputs: a slot is free again once its unit's readout MMA and copy-out
// are done, so the next unit's loads stream in while the current one computes. All waits are
// bounded.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "m3_common.cuh"
#include "m3_internal.h"
#include "m3_sm100.cuh"

namespace m3 {
namespace {

using namespace sm100;

constexpr int kThreads = 256;
constexpr int kN = 128, kP = 64, kHalf = 64;
constexpr int kRing = 2;

// Shared-memory layout (bytes after 1024-byte alignment).
template <int R>
struct DecCfg {
    static constexpr uint32_t HB = 0;                   // fp32 state tiles x2: two boxes of
    static constexpr uint32_t H_BYTES = 32768;          // 128 rows x 32 columns each
    static constexpr uint32_t AU = kRing * H_BYTES;     // A of U: [n][k] bf16, K-major SW32
    static constexpr uint32_t BU = AU + 4096;           // B of U: [p][k] bf16, K-major SW32
    static constexpr uint32_t CB = BU + 2048;           // B of y: [r][n] fp32, K-major SW128
    static constexpr uint32_t SM0 = CB + 4096;          // small inputs ring
    // one small-input slot: x, x_prev [R][P]; B, C, B_prev [R][N]; theta [N/2] bf16; phi [N/2]
    static constexpr uint32_t S_X = 0, S_XP = S_X + R * kP * 2, S_B = S_XP + R * kP * 2,
                              S_C = S_B + R * kN * 2, S_BP = S_C + R * kN * 2,
                              S_TH = S_BP + R * kN * 2, S_PHI = S_TH + kHalf * 2,
                              S_Z = S_PHI + kHalf * 4,   // z' [P] (projected decode)
                              S_W = S_Z + kP * 2,        // the head's W_X, W_Z, W_O [R][P] fp32
                              S_BYTES = (S_W + 3 * R * kP * 4 + 127) / 128 * 128;
    static constexpr uint32_t SCR = SM0 + kRing * S_BYTES;  // fp32 scratch
    static constexpr uint32_t TOTAL = SCR + 4 * (3 * 8 + 4 * kRing) + 1024;
    static constexpr uint32_t TX = 2 * 16384 + 2 * R * kP * 2 + 3 * R * kN * 2 + kHalf * 2 + kHalf * 4;
    // projected decode: x' and z' [P] in place of x [R][P]
    static constexpr uint32_t TX_PROJ = TX - R * kP * 2 + 2 * kP * 2 + 3 * R * kP * 4;
};
constexpr uint32_t kTmemCols = 128;
constexpr uint32_t T_U = 0, T_Y = 64;

struct DecMaps {
    CUtensorMap h0;
};

__device__ __forceinline__ float reduce_turns(float x) {
    // x reduced by a whole number of turns into [-pi, pi] (Cody & Waite's two-constant
    // reduction, "Software Manual for the Elementary Functions", 1980)
    const float k = rintf(x * 0.15915494309189535f);
    return fmaf(-k, 1.9353071795864769e-3f, fmaf(-k, 6.28125f, x));
}
__device__ __forceinline__ uint32_t pack2(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ void tmem_ld_32x32b_x8(uint32_t taddr, float (&v)[8]) {
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}
// Bulk copy of bytes (a multiple of 16, both addresses 16-byte aligned) from shared to global
// memory, in this thread's current bulk async-group.
__device__ __forceinline__ void bulk_store(void* gdst, const void* ssrc, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                 :: "l"(gdst), "r"(smem_u32(ssrc)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Waits until this thread's bulk copies have read their sources (shared memory reusable) ...
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// ... or have completed (global writes done).
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// Byte offset of bf16 element (row, col) in a K-major tile with 32-byte rows and the 32-byte
// swizzle (16-byte chunk c of row r stored at chunk c ^ ((r / 4) mod 2)).
__device__ __forceinline__ uint32_t swz32(uint32_t row, uint32_t col) {
    return row * 32u + ((((col >> 3) ^ (row >> 2)) & 1u) << 4) + ((col & 7u) << 1);
}
// Byte offset of fp32 element (row, col) in one 32-column slab of a 128-byte swizzled tile.
__device__ __forceinline__ uint32_t swz128_f32(uint32_t row, uint32_t col) {
    return row * 128u + ((((col >> 2) ^ row) & 7u) << 4) + ((col & 3u) << 2);
}
// High half of a shared-memory descriptor with the 32-byte swizzle (layout type 6).
__host__ __device__ constexpr uint32_t desc_hi_sw32(uint32_t sbo_bytes) {
    return (sbo_bytes >> 4) | (1u << 14) | (6u << 29);
}
// Instruction descriptor: tf32 x tf32 -> fp32, dense.
__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N, bool a_mn_major, bool b_mn_major) {
    return (1u << 4) | (2u << 7) | (2u << 10) | (static_cast<uint32_t>(a_mn_major) << 15) |
           (static_cast<uint32_t>(b_mn_major) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
           (static_cast<uint32_t>(M >> 4) << 24);
}
__device__ __forceinline__ void mma_tf32(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n"
        :
        : "r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(accumulate));
}
// R consecutive bf16 values into row n of a K-major SW32 tile, columns [k0, k0 + R)
// (k0 + R <= 16, k0 a multiple of R).
template <int R>
__device__ __forceinline__ void store_kvec(uint8_t* tile, int n, int k0, const float (&v)[R]) {
    uint8_t* dst = tile + swz32(n, k0);
    if constexpr (R == 8) {
        *reinterpret_cast<uint4*>(dst) = make_uint4(pack2(v[0], v[1]), pack2(v[2], v[3]),
                                                    pack2(v[4], v[5]), pack2(v[6], v[7]));
    } else if constexpr (R == 4) {
        *reinterpret_cast<uint2*>(dst) = make_uint2(pack2(v[0], v[1]), pack2(v[2], v[3]));
    } else if constexpr (R == 2) {
        *reinterpret_cast<uint32_t*>(dst) = pack2(v[0], v[1]);
    } else {
        *reinterpret_cast<__nv_bfloat16*>(dst) = __float2bfloat16_rn(v[0]);
    }
}

// kRaw: dt and lam arrive raw (m3_dims.flags); the step scalars apply softplus / sigmoid.
// kProj: the MIMO projections (Appendix C): x' and z' [P] in, X = W_X x' expanded here and
// kept as the stored previous token, O' = sum_r W_O Y SiLU(W_Z z') out.
template <int R, bool kRaw, bool kProj>
__global__ void __launch_bounds__(kThreads, 2)
decode_tc_kernel(const ScanParams p, const __grid_constant__ DecMaps maps, const int n_units) {
    using Cfg = DecCfg<R>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    float* rs = reinterpret_cast<float*>(sm + Cfg::SCR);      // [3R] RMS scales
    float* scal = rs + 3 * 8;                                 // [ring][4]: dt, A, lam
    __shared__ uint64_t bar_full[kRing], bar_u, bar_y;
    __shared__ uint32_t tslot;
    __shared__ int s_abort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const __nv_bfloat16* xg = static_cast<const __nv_bfloat16*>(p.x);
    const __nv_bfloat16* Bg = static_cast<const __nv_bfloat16*>(p.B);
    const __nv_bfloat16* Cg = static_cast<const __nv_bfloat16*>(p.C);
    const __nv_bfloat16* thg = static_cast<const __nv_bfloat16*>(p.theta);
    const __nv_bfloat16* pBg = static_cast<const __nv_bfloat16*>(p.prevB0);
    const __nv_bfloat16* pxg = static_cast<const __nv_bfloat16*>(p.prevx0);

    // every input of unit u into ring slot s (one thread)
    auto issue = [&](int u, int s) {
        uint8_t* sl = sm + Cfg::SM0 + s * Cfg::S_BYTES;
        uint8_t* hb = sm + Cfg::HB + s * Cfg::H_BYTES;
        const int64_t bb = u / p.H, hh = u % p.H, g = hh / (p.H / p.G);
        uint64_t* bar = &bar_full[s];
        mbar_arrive_expect_tx(bar, kProj ? Cfg::TX_PROJ : Cfg::TX);
        tma_load_3d(hb, &maps.h0, bar, 0, 0, u);
        tma_load_3d(hb + 16384, &maps.h0, bar, 32, 0, u);
        if constexpr (kProj) {
            bulk_load(sl + Cfg::S_X, static_cast<const __nv_bfloat16*>(p.xprj) + static_cast<int64_t>(u) * kP,
                      kP * 2, bar);
            bulk_load(sl + Cfg::S_Z, static_cast<const __nv_bfloat16*>(p.zprj) + static_cast<int64_t>(u) * kP,
                      kP * 2, bar);
            // the head's weights ride with the unit: consecutive units are different heads
            bulk_load(sl + Cfg::S_W, p.WX + hh * R * kP, R * kP * 4, bar);
            bulk_load(sl + Cfg::S_W + R * kP * 4, p.WZ + hh * R * kP, R * kP * 4, bar);
            bulk_load(sl + Cfg::S_W + 2 * R * kP * 4, p.WO + hh * R * kP, R * kP * 4, bar);
        } else {
            bulk_load(sl + Cfg::S_X, xg + static_cast<int64_t>(u) * R * kP, R * kP * 2, bar);
        }
        bulk_load(sl + Cfg::S_XP, pxg + static_cast<int64_t>(u) * R * kP, R * kP * 2, bar);
        bulk_load(sl + Cfg::S_B, Bg + (bb * p.G + g) * R * kN, R * kN * 2, bar);
        bulk_load(sl + Cfg::S_C, Cg + (bb * p.G + g) * R * kN, R * kN * 2, bar);
        bulk_load(sl + Cfg::S_BP, pBg + static_cast<int64_t>(u) * R * kN, R * kN * 2, bar);
        bulk_load(sl + Cfg::S_TH, thg + static_cast<int64_t>(u) * kHalf, kHalf * 2, bar);
        bulk_load(sl + Cfg::S_PHI, p.phi0 + static_cast<int64_t>(u) * kHalf, kHalf * 4, bar);
    };

    // thread 0: loads issued into each ring slot and how many of them were waited for
    int issued[kRing] = {0, 0}, waited[kRing] = {0, 0};
    int u = blockIdx.x;
    if (tid == 0) {
        for (int s = 0; s < kRing; ++s) mbar_init(&bar_full[s], 1);
        mbar_init(&bar_u, 1);
        mbar_init(&bar_y, 2);   // one commit per half of the readout
        fence_mbar_init();
        s_abort = 0;
        if (u < n_units) {
            issue(u, 0);
            ++issued[0];
            scal[0] = step_dt<kRaw>(p.dt[u], (kRaw && p.dt_bias) ? p.dt_bias[u % static_cast<int>(p.H)] : 0.f,
                                    p.flags);
            scal[1] = p.A[u];
            scal[2] = step_lam<kRaw>(p.lam[u], p.flags);
        }
    }
    if (warp == 0) tmem_alloc(&tslot, kTmemCols);
    // operand columns never written per unit stay zero: A_U and B_U beyond column 2R, C
    // rows beyond R
    for (int i = tid; i < (4096 + 2048 + 4096) / 16; i += kThreads)  // AU, BU, CB are contiguous
        *reinterpret_cast<uint4*>(sm + Cfg::AU + 16 * i) = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = tslot;
    const uint32_t id_u = idesc_bf16(128, 64, false, false);   // U = A_U . B_U^T
    const uint32_t id_y = idesc_tf32(64, 8, true, false);      // y^T = h'^T . C^T

    uint32_t mma_phase = 0;
    for (int i = 0; u < n_units; ++i, u += gridDim.x) {
        const int s = i % kRing;
        // the next unit's dt, A, lam: loaded into registers now, stored to its slot after this
        // unit's state update (raw scalars transformed there), so the load latency is spent on
        // this unit's work
        float snext[4] = {0.f, 0.f, 0.f, 0.f};   // dt, A, lam, dt bias
        uint8_t* sl = sm + Cfg::SM0 + s * Cfg::S_BYTES;
        uint8_t* hb = sm + Cfg::HB + s * Cfg::H_BYTES;
        if (tid == 0) {
            // the other slot held the previous unit, whose readout and copy-out have finished:
            // it takes the next unit, which then streams in while this one computes
            const int un = u + static_cast<int>(gridDim.x);
            bulk_wait_read();   // the previous unit's stored-token copies have left its slot
            if (un < n_units) {
                issue(un, s ^ 1);
                ++issued[s ^ 1];
                snext[0] = p.dt[un];
                snext[1] = p.A[un];
                snext[2] = p.lam[un];
                if constexpr (kRaw) snext[3] = p.dt_bias ? p.dt_bias[un % static_cast<int>(p.H)] : 0.f;
            }
            if (mbar_wait_sleep(&bar_full[s], static_cast<uint32_t>((i / kRing) & 1))) ++waited[s];
            else s_abort = 1;
        }
        __syncthreads();
        if (s_abort) break;
        (void)mbar_try_wait(smem_u32(&bar_full[s]), static_cast<uint32_t>((i / kRing) & 1));

        const __nv_bfloat16* sB = reinterpret_cast<const __nv_bfloat16*>(sl + Cfg::S_B);
        const __nv_bfloat16* sC = reinterpret_cast<const __nv_bfloat16*>(sl + Cfg::S_C);
        const __nv_bfloat16* sBp = reinterpret_cast<const __nv_bfloat16*>(sl + Cfg::S_BP);
        const __nv_bfloat16* sx = reinterpret_cast<const __nv_bfloat16*>(sl + Cfg::S_X);
        const __nv_bfloat16* sxp = reinterpret_cast<const __nv_bfloat16*>(sl + Cfg::S_XP);
        const float d = scal[4 * s + 0], a = scal[4 * s + 1], lm = scal[4 * s + 2];
        const float al = __expf(d * a);
        float be = (1.f - lm) * d * al, ga = lm * d;
        if constexpr (kRaw) {
            if (p.flags & 4u) {   // zero-order hold: no previous-token term
                be = 0.f;
                ga = zoh_gamma(d, a);
            }
        }
        const int64_t hh = u % p.H;

        // ---- RMS scales of B, C and the stored previous B, one warp per vector ----
        if (p.bc_norm) {
            for (int v = warp; v < 3 * R; v += kThreads / 32) {
                const __nv_bfloat16* src = (v < R) ? sB + v * kN : (v < 2 * R) ? sC + (v - R) * kN
                                                                             : sBp + (v - 2 * R) * kN;
                const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(src + 2 * lane));
                const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(src + 64 + 2 * lane));
                float ss = fmaf(f0.x, f0.x, fmaf(f0.y, f0.y, fmaf(f1.x, f1.x, f1.y * f1.y)));
                ss = warp_sum(ss);
                if (lane == 0) rs[v] = rsqrtf(ss / static_cast<float>(kN) + p.eps);
            }
            __syncthreads();
        }

        // ---- operand tiles: thread (role, pair i) ----
        {
            const int role = tid >> 6, i = tid & 63;
            if (role < 3) {
                // role 0: B by the new angle (gamma), 1: B_prev by the old one (beta), 2: C by
                // the new angle; pair (i, i + N/2)
                const float ph_old = reinterpret_cast<const float*>(sl + Cfg::S_PHI)[i];
                const float th = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(sl + Cfg::S_TH)[i]);
                const float ph = role == 1 ? ph_old : ph_old + d * th;
                if (role == 0 && p.phi1) p.phi1[static_cast<int64_t>(u) * kHalf + i] = ph;
                float sn, cn;
                __sincosf(reduce_turns(ph), &sn, &cn);
                const __nv_bfloat16* src = role == 0 ? sB : role == 1 ? sBp : sC;
                const float* bias = role == 2 ? p.Cbias : p.Bbias;
                const float scale = role == 0 ? ga : role == 1 ? be : 1.f;
                const int rsb = role == 0 ? 0 : role == 1 ? 2 * R : R;
                float v0[R], v1[R];
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const float b0 = bias ? bias[(hh * R + r) * kN + i] : 0.f;
                    const float b1 = bias ? bias[(hh * R + r) * kN + i + kHalf] : 0.f;
                    const float sr = p.bc_norm ? rs[rsb + r] : 1.f;
                    const float u0 = fmaf(__bfloat162float(src[r * kN + i]), sr, b0);
                    const float u1 = fmaf(__bfloat162float(src[r * kN + i + kHalf]), sr, b1);
                    v0[r] = scale * (u0 * cn + u1 * sn);
                    v1[r] = scale * (u1 * cn - u0 * sn);
                }
                if (role < 2) {
                    // A_U rows i and i + N/2: columns [0, R) beta Bbar_prev, [R, 2R) gamma Bbar
                    const int k0 = role == 1 ? 0 : R;
                    store_kvec<R>(sm + Cfg::AU, i, k0, v0);
                    store_kvec<R>(sm + Cfg::AU, i + kHalf, k0, v1);
                } else {
                    // C^T as the K-major fp32 B of the readout: row r, column n, four 32-column
                    // slabs of 8 rows x 128 B
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        *reinterpret_cast<float*>(sm + Cfg::CB + (i >> 5) * 1024 + swz128_f32(r, i & 31)) = v0[r];
                        *reinterpret_cast<float*>(sm + Cfg::CB + ((i + kHalf) >> 5) * 1024 + swz128_f32(r, i & 31)) = v1[r];
                    }
                }
            } else {
                // B_U row p = i: columns [0, R) x_prev[r][p], [R, 2R) x[r][p]
                float vp[R], vx[R];
#pragma unroll
                for (int r = 0; r < R; ++r) vp[r] = __bfloat162float(sxp[r * kP + i]);
                if constexpr (kProj) {
                    // X[r][p] = W_X[h][r][p] x'[p]; written over x' (this thread alone reads
                    // x'[p]) as the stored previous token, which is bulk-copied from there
                    const float xin = __bfloat162float(sx[i]);
                    const float* sw = reinterpret_cast<const float*>(sl + Cfg::S_W) + i;
                    __nv_bfloat16* sxw = reinterpret_cast<__nv_bfloat16*>(sl + Cfg::S_X);
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        vx[r] = sw[r * kP] * xin;
                        sxw[r * kP + i] = __float2bfloat16_rn(vx[r]);
                    }
                } else {
#pragma unroll
                    for (int r = 0; r < R; ++r) vx[r] = __bfloat162float(sx[r * kP + i]);
                }
                store_kvec<R>(sm + Cfg::BU, i, 0, vp);
                store_kvec<R>(sm + Cfg::BU, i, R, vx);
            }
        }
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();
        fence_after_sync();
        // ---- U = A_U B_U^T: one K = 16 step covers the 2R <= 16 columns ----
        if (warp == 0) {
            if (elect_one()) {
                constexpr uint32_t hi32 = desc_hi_sw32(256);   // 8-row groups of 32-byte rows
                mma_bf16(tmem + T_U, desc_pack(desc_lo(smem_u32(sm + Cfg::AU), 16), hi32),
                         desc_pack(desc_lo(smem_u32(sm + Cfg::BU), 16), hi32), id_u, 0u);
                mma_commit(smem_u32(&bar_u));
            }
            __syncwarp();
        }
        if constexpr (kProj) {
            // the output weights of Y[r][p], independent of Y: g = W_O SiLU(W_Z z'), written
            // over W_Z by all threads while the update MMA runs (read after the next barrier)
            float* sw = reinterpret_cast<float*>(sl + Cfg::S_W);
            const __nv_bfloat16* sz = reinterpret_cast<const __nv_bfloat16*>(sl + Cfg::S_Z);
#pragma unroll
            for (int e = tid; e < R * kP; e += kThreads) {
                const int r = e / kP, pc = e % kP;
                const float z = sw[(R + r) * kP + pc] * __bfloat162float(sz[pc]);
                sw[(R + r) * kP + pc] = sw[(2 * R + r) * kP + pc] * z * __frcp_rn(1.f + __expf(-z));
            }
        }
        if (!mbar_wait(&bar_u, mma_phase)) s_abort = 1;
        fence_after_sync();
        // ---- h' = alpha h + U: state row n = 32 q + lane, columns [32 wh, 32 wh + 32) ----
        {
            const int q = warp & 3, wh = warp >> 2, n = 32 * q + lane;
            float uv[32];
            {
                float t0[16], t1[16];
                const uint32_t ta = tmem + ((32u * q) << 16) + T_U + 32u * wh;
                tmem_ld_32x32b_x16(ta, t0);
                tmem_ld_32x32b_x16(ta + 16, t1);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) { uv[j] = t0[j]; uv[16 + j] = t1[j]; }
            }
            uint8_t* hrow = hb + wh * 16384 + n * 128;
#pragma unroll
            for (int j = 0; j < 8; ++j) {  // 16-byte piece j: half (j mod 2) of 32-byte chunk j / 2
                float4* ptr = reinterpret_cast<float4*>(hrow + (((((j >> 1) ^ n) & 3) << 5) | ((j & 1) << 4)));
                float4 h = *ptr;
                h.x = fmaf(al, h.x, uv[4 * j]);
                h.y = fmaf(al, h.y, uv[4 * j + 1]);
                h.z = fmaf(al, h.z, uv[4 * j + 2]);
                h.w = fmaf(al, h.w, uv[4 * j + 3]);
                *ptr = h;
            }
        }
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();
        fence_after_sync();
        if (warp == 0 || warp == 4) {
            if (elect_one()) {
                // ---- y^T = h'^T C^T in tf32: A = the fp32 state tile, MN-major (rows n = K in
                // 4-row atoms of 512 B, 32-column boxes 16 KB apart = M blocks); B = C^T, K-major
                // with the plain 128-byte swizzle; K steps of 8 rows. Two warps issue one half of
                // the K range each, into two accumulators that the readout adds. ----
                constexpr uint32_t hiA = (512u >> 4) | (1u << 14) | (1u << 29);  // layout type 1
                constexpr uint32_t hiB = desc_hi_sw128(1024);
                const uint32_t loA = desc_lo(smem_u32(hb), 16384), loB = desc_lo(smem_u32(sm + Cfg::CB), 16);
                const int k0 = warp == 0 ? 0 : 8;
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_tf32(tmem + T_Y + (warp == 0 ? 0u : 8u), desc_pack(loA + ((1024u * (k0 + k)) >> 4), hiA),
                             desc_pack(loB + (kmajor_off(k0 + k, 1024) >> 4), hiB), id_y, k > 0);
                mma_commit(smem_u32(&bar_y));
            }
            __syncwarp();
        }
        // the next unit's step scalars (softplus / sigmoid of raw ones) into its slot, which no
        // one reads during this unit; here their loads have long landed and the work overlaps
        // the copy-out and the readout instead of delaying the unit's last barrier
        if (tid == 0) {
            scal[4 * (s ^ 1) + 0] = step_dt<kRaw>(snext[0], snext[3], p.flags);
            scal[4 * (s ^ 1) + 1] = snext[1];
            scal[4 * (s ^ 1) + 2] = step_lam<kRaw>(snext[2], p.flags);
        }
        // ---- the updated state to HBM: consecutive threads take consecutive 16-byte pieces of
        // the [N][P] row-major state (piece c of row n: box c / 8, 32-byte chunk (c mod 8) / 2)
        {
            float4* dst = reinterpret_cast<float4*>(p.h1 + static_cast<int64_t>(u) * kN * kP);
#pragma unroll
            for (int k = 0; k < kN * kP / 4 / kThreads; ++k) {
                const int e = tid + k * kThreads;          // 16-byte piece of the unit's state
                const int n = e >> 4, c = e & 15, box = c >> 3, j = c & 7;
                dst[e] = *reinterpret_cast<const float4*>(hb + box * 16384 + n * 128 +
                                                          (((((j >> 1) ^ n) & 3) << 5) | ((j & 1) << 4)));
            }
        }
        // last token's raw B and x become the stored previous token: two bulk copies from the
        // slot, by one thread (waited for before the slot is refilled)
        if (tid == 0) {
            if (p.prevB1)
                bulk_store(static_cast<__nv_bfloat16*>(p.prevB1) + static_cast<int64_t>(u) * R * kN, sB, R * kN * 2);
            if (p.prevx1)
                bulk_store(static_cast<__nv_bfloat16*>(p.prevx1) + static_cast<int64_t>(u) * R * kP, sx, R * kP * 2);
            bulk_commit();
        }
        if (!mbar_wait(&bar_y, mma_phase)) s_abort = 1;
        fence_after_sync();
        mma_phase ^= 1;
        // ---- y: accumulator row p sits in lane (p mod 16) + 32 (p / 16), column r ----
        if (warp < 4) {
            float yv[8], yw[8];
            tmem_ld_32x32b_x8(tmem + ((32u * warp) << 16) + T_Y, yv);
            tmem_ld_32x32b_x8(tmem + ((32u * warp) << 16) + T_Y + 8, yw);
            tmem_wait_ld();
#pragma unroll
            for (int r = 0; r < 8; ++r) yv[r] += yw[r];
            if (lane < 16) {
                const int pcol = 16 * warp + lane;
                if constexpr (kProj) {
                    // O'[p] = sum_r W_O[h][r][p] SiLU(W_Z[h][r][p] z'[p]) Y[r][p], the gate
                    // factors formed while the update MMA ran
                    const float* gw = reinterpret_cast<const float*>(sl + Cfg::S_W) + R * kP + pcol;
                    float o = 0.f;
#pragma unroll
                    for (int r = 0; r < R; ++r) o = fmaf(gw[r * kP], yv[r], o);
                    static_cast<__nv_bfloat16*>(p.y)[static_cast<int64_t>(u) * kP + pcol] = __float2bfloat16_rn(o);
                } else {
                    __nv_bfloat16* yo = static_cast<__nv_bfloat16*>(p.y) + static_cast<int64_t>(u) * R * kP + pcol;
#pragma unroll
                    for (int r = 0; r < R; ++r) yo[r * kP] = __float2bfloat16_rn(yv[r]);
                }
            }
        }
        fence_before_sync();
        __syncthreads();
        fence_after_sync();
    }
    if (tid == 0) {
        bulk_wait_all();
        if (s_abort && p.status) atomicExch(p.status, 1);
        // inputs requested but never waited for (only after a wait gave up): let them land
        for (int h = 0; h < kRing; ++h)
            for (int k = waited[h]; k < issued[h]; ++k)
                (void)mbar_wait(&bar_full[h], static_cast<uint32_t>(k & 1), 200000000LL);
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

// fp32 state [units][N][P] as 3D (P, N, units), boxes of 32 columns x 128 rows, 128-byte
// swizzle of 32-byte atoms
bool encode_state(CUtensorMap* m, const float* base, int64_t units) {
    auto enc = get_encode();
    if (!enc) return false;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kP), static_cast<cuuint64_t>(kN),
                                static_cast<cuuint64_t>(units)};
    const cuuint64_t str[2] = {kP * 4, static_cast<cuuint64_t>(kN) * kP * 4};
    const cuuint32_t box[3] = {32, static_cast<cuuint32_t>(kN), 1};
    const cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), dims, str, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int R>
cudaError_t launch_tc_t(const ScanParams& p, cudaStream_t s) {
    const int sms = device_sm_count();
    const int64_t units = p.b * p.H;
    DecMaps maps;
    if (!encode_state(&maps.h0, p.h0, units)) return cudaErrorInvalidValue;
    const uint32_t smem = DecCfg<R>::TOTAL;
    auto k = p.proj ? (p.flags ? decode_tc_kernel<R, true, true> : decode_tc_kernel<R, false, true>)
                    : (p.flags ? decode_tc_kernel<R, true, false> : decode_tc_kernel<R, false, false>);
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const int grid = units < 2 * sms ? static_cast<int>(units) : 2 * sms;
    k<<<grid, kThreads, smem, s>>>(p, maps, static_cast<int>(units));
    return cudaGetLastError();
}

}  // namespace

// Used for ranks 4 and 8, where the rank-2R arithmetic would bound the CUDA-core form; at
// ranks 1 and 2 the bulk-copy kernel, whose per-unit latency chain is shorter, is faster.
bool decode_tc_supported(const ScanParams& p, bool bf16) {
    return bf16 && p.N == kN && p.P == kP && (p.R == 4 || p.R == 8) &&
           p.b * p.H < (int64_t(1) << 31) && p.h0 && p.h1;
}

cudaError_t launch_decode_tc(const ScanParams& p, cudaStream_t s) {
    switch (p.R) {
        case 4: return launch_tc_t<4>(p, s);
        case 8: return launch_tc_t<8>(p, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace m3
