// The state at the start of a sequence segment from the end states of the segments before it,
// for prefill split over devices along the sequence (context parallelism).
//
// The recurrence is linear in the state ("Mamba-3: Improved Sequence Modeling using State
// Space Principles", Sec. 3.1.1 Prop. 1) and its rotated frame is an accumulated rotation of
// B and C (Sec. 3.2.2 Prop. 4), so a segment run from zero with angle 0 at its start (and the
// previous segment's last token folded in) contributes its end state, rotated by the true
// angle at its start, on top of the earlier state decayed by the segment's summed log-decay:
//     h <- e^{Lambda_j} h + R(-phi_j) dH_j,   phi_{j+1} = phi_j + (segment j's angle sum),
// starting from segment 0's end state, which was run from the true initial state. R(-phi)
// acts on the rotation pairs (i, i + N/2): v_i cos + v_{i+N/2} sin, -v_i sin + v_{i+N/2} cos.
#include "m3_common.cuh"
#include "m3_internal.h"

namespace m3 {
namespace {

constexpr int kCombineThreads = 256;

// One CTA per (batch, head) unit; threads over the N x P state elements. Segment j of unit u
// sits at h + j * seg_stride + u * unit_stride (phi and lam at their own offsets from there).
__global__ void __launch_bounds__(kCombineThreads)
state_combine_kernel(int64_t units, int N, int P, int nseg, SegSrc src,
                     float* __restrict__ h_out, float* __restrict__ phi_out,
                     float* __restrict__ lam_out) {
    const int64_t u = blockIdx.x;
    const int half = N / 2;
    auto hp = [&](int j) { return src.h + j * src.h_seg + u * src.h_unit; };
    auto pp = [&](int j) { return src.phi + j * src.phi_seg + u * src.phi_unit; };
    auto lp = [&](int j) { return src.lam[j * src.lam_seg + u * src.lam_unit]; };
    for (int e = threadIdx.x; e < N * P; e += blockDim.x) {
        const int n = e / P, col = e % P, i = n % half;
        const int other = n < half ? n + half : n - half;
        float h = hp(0)[e];
        float phi = pp(0)[i];
        for (int j = 1; j < nseg; ++j) {
            float sn, cs;
            sincosf(phi, &sn, &cs);
            const float own = hp(j)[e];
            const float oth = hp(j)[other * P + col];
            const float rot = n < half ? own * cs + oth * sn : own * cs - oth * sn;
            h = fmaf(expf(lp(j)), h, rot);
            phi += pp(j)[i];
        }
        h_out[u * N * P + e] = h;
    }
    for (int i = threadIdx.x; i < half; i += blockDim.x) {
        float phi = pp(0)[i];
        for (int j = 1; j < nseg; ++j) phi += pp(j)[i];
        phi_out[u * half + i] = phi;
    }
    if (lam_out && threadIdx.x == 0) {
        float l = 0.f;
        for (int j = 0; j < nseg; ++j) l += lp(j);
        lam_out[u] = l;
    }
}

}  // namespace

cudaError_t launch_state_combine(int64_t units, int N, int P, int nseg, const SegSrc& src,
                                 float* h_out, float* phi_out, float* lam_out, cudaStream_t s) {
    if (units == 0) return cudaSuccess;
    state_combine_kernel<<<static_cast<unsigned>(units), kCombineThreads, 0, s>>>(
        units, N, P, nseg, src, h_out, phi_out, lam_out);
    return cudaGetLastError();
}

}  // namespace m3
