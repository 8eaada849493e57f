// gs_train.cu -- the training step's own kernels: Adam fused with the sum of
// the gradient slots, the step counter, and the per-camera L1 loss that also
// records the camera's binning status.
//
// Source: "Gaussian splatting in PyTorch" s7 (render, L1 against the target,
// backward, torch.optim.Adam over the raw parameters with a learning rate
// per group); Adam is Kingma and Ba's algorithm, evaluated in the form torch
// uses: p -= (lr / (1 - b1^t)) m / (sqrt(v) / sqrt(1 - b2^t) + eps).
//
// Adam is a streaming update: per value it reads p, m, v and one value per
// gradient slot and writes p, m, v (and g when asked), so it is bound by
// HBM bandwidth.  One launch covers the five parameter groups (blockIdx.y);
// each group's arrays are walked as float4 where every array of the group is
// 16-byte aligned, with a scalar tail.
#include <cmath>

#include "gs_internal.cuh"

namespace gs {
namespace {

// Bias corrections of step t, in double precision (1 - 0.999^t loses half
// its digits in single precision for small t).
struct AdamStepConsts {
    float step_size;    // lr / (1 - beta1^t), per group
    float inv_sqrt_bc2; // 1 / sqrt(1 - beta2^t)
};

__device__ __forceinline__ float4 ld4(const float *p, int64_t i) {
    return reinterpret_cast<const float4 *>(p)[i];
}
__device__ __forceinline__ void st4(float *p, int64_t i, float4 v) { reinterpret_cast<float4 *>(p)[i] = v; }

__device__ __forceinline__ float adam_one(float &p, float &m, float &v, float g, const AdamBetas &B,
                                          float eps, float step_size, float inv_sqrt_bc2) {
    m = __fmaf_rn(B.b1f, m, B.omb1 * g);
    v = __fmaf_rn(B.b2f, v, B.omb2 * g * g);
    const float denom = __fadd_rn(__fmul_rn(__fsqrt_rn(v), inv_sqrt_bc2), eps);
    p = __fsub_rn(p, __fdiv_rn(__fmul_rn(step_size, m), denom));
    return g;
}

// kUpdate false: only g = grad_scale * sum of slots is written to A.out.
template <int kMaxSlots, bool kUpdate>
__global__ void __launch_bounds__(256)
k_adam(AdamGroups G, AdamBetas B, float eps, float grad_scale, int n_slots, const int64_t *__restrict__ step) {
    const AdamGroup &A = G.g[blockIdx.y];
    __shared__ AdamStepConsts s_c;
    if (kUpdate && threadIdx.x == 0) {
        const double t = (double)(*step);  // already advanced by k_adam_tick
        const double bc1 = 1.0 - pow(B.b1, t), bc2 = 1.0 - pow(B.b2, t);
        s_c.step_size = (float)((double)A.lr / bc1);
        s_c.inv_sqrt_bc2 = (float)(1.0 / sqrt(bc2));
    }
    __syncthreads();
    const float ss = kUpdate ? s_c.step_size : 0.f, ib = kUpdate ? s_c.inv_sqrt_bc2 : 0.f;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t i0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    int64_t done = 0;
    if (A.vec) {
        const int64_t nv = A.count / 4;
        for (int64_t i = i0; i < nv; i += stride) {
            float4 g = ld4(A.slot[0], i);
#pragma unroll
            for (int s = 1; s < kMaxSlots; s++) {
                if (s >= n_slots) break;
                const float4 h = ld4(A.slot[s], i);
                g.x += h.x; g.y += h.y; g.z += h.z; g.w += h.w;
            }
            g.x *= grad_scale; g.y *= grad_scale; g.z *= grad_scale; g.w *= grad_scale;
            if (A.out) st4(A.out, i, g);
            if (!kUpdate) continue;
            float4 p = ld4(A.p, i), m = ld4(A.m, i), v = ld4(A.v, i);
            adam_one(p.x, m.x, v.x, g.x, B, eps, ss, ib);
            adam_one(p.y, m.y, v.y, g.y, B, eps, ss, ib);
            adam_one(p.z, m.z, v.z, g.z, B, eps, ss, ib);
            adam_one(p.w, m.w, v.w, g.w, B, eps, ss, ib);
            st4(A.p, i, p);
            st4(A.m, i, m);
            st4(A.v, i, v);
        }
        done = nv * 4;
    }
    for (int64_t i = done + i0; i < A.count; i += stride) {
        float g = A.slot[0][i];
        for (int s = 1; s < n_slots; s++) g += A.slot[s][i];
        g *= grad_scale;
        if (A.out) A.out[i] = g;
        if (!kUpdate) continue;
        float p = A.p[i], m = A.m[i], v = A.v[i];
        adam_one(p, m, v, g, B, eps, ss, ib);
        A.p[i] = p;
        A.m[i] = m;
        A.v[i] = v;
    }
}

// Advances the device step counter before the update reads it.
__global__ void k_adam_tick(int64_t *step) { *step += 1; }

int num_sms_train() {
    static int sms = 0;
    if (sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (sms <= 0) sms = 148;
    }
    return sms;
}

}  // namespace

cudaError_t launch_adam(const AdamGroups &G, int64_t max_count, const AdamBetas &B, float eps,
                        float grad_scale, int n_slots, int64_t *step, cudaStream_t s, bool update) {
    prof_before(update ? "adam" : "grad_sum", s);
    int kernels = 0;
    if (update) {
        k_adam_tick<<<1, 1, 0, s>>>(step);
        kernels++;
    }
    if (max_count > 0) {
        const int64_t want = (max_count / 4 + 255) / 256;
        const int64_t cap = (int64_t)num_sms_train() * 8;
        const unsigned bx = (unsigned)std::max<int64_t>(1, std::min(want, cap));
        if (update)
            k_adam<kAdamMaxSlots, true><<<dim3(bx, 5), 256, 0, s>>>(G, B, eps, grad_scale, n_slots, step);
        else
            k_adam<kAdamMaxSlots, false><<<dim3(bx, 5), 256, 0, s>>>(G, B, eps, grad_scale, n_slots, step);
        kernels++;
    }
    prof_after(s, kernels);
    return cudaGetLastError();
}


}  // namespace gs
