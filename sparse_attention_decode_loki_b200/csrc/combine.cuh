// Log-sum-exp merge of split partials (flash-decoding style), shared by the
// sparse and the dense attention kernels.
//
// A partial is (m, l, acc[D]) in the base-2 domain: m the running max of
// scale*log2(e)*score, l = sum 2^(a_j - m), acc = sum 2^(a_j - m) V_j. Partial
// slots are grouped by work unit: slot((unit, part), g) = (unit * maxp + part)
// * Gc + g, where a unit is a (batch, query head) row for sparse attention
// (Gc = 1) and a (batch, KV head) for dense attention (Gc = G query heads).
// Units own `items` consecutive work items of a static split in which CTA c
// owns items [c * per, (c + 1) * per); part = CTA index - first CTA of the unit.
#pragma once

#include "common.cuh"

namespace loki {

template <class E>
__global__ void __launch_bounds__(128) k_combine(const float2* __restrict__ part_ml,
                                                 const float* __restrict__ part_acc,
                                                 typename E::T* __restrict__ out, int H_q, int Gc,
                                                 int64_t items, int64_t per, int maxp, int D) {
    const int64_t r = blockIdx.x;
    const int b = (int)(r / H_q), h = (int)(r % H_q);
    const int64_t unit = (int64_t)b * (H_q / Gc) + h / Gc;
    const int g = h % Gc;
    const int64_t c0 = (unit * items) / per;
    const int64_t c1 = (unit * items + items - 1) / per;
    const int np = (int)(c1 - c0 + 1);
    const int c = threadIdx.x;
    griddep_wait();  // partials come from the attention kernel
    griddep_launch_dependents();
    float M = -INFINITY;
    for (int p = 0; p < np; ++p) M = fmaxf(M, part_ml[(unit * maxp + p) * Gc + g].x);
    float L = 0.f, A = 0.f;
    if (M != -INFINITY) {
        for (int p = 0; p < np; ++p) {
            const int64_t slot = (unit * maxp + p) * Gc + g;
            const float2 ml = part_ml[slot];
            const float sc = exp2f(ml.x - M);
            L += ml.y * sc;
            if (c < D) A += part_acc[slot * D + c] * sc;
        }
    }
    if (c < D) out[r * D + c] = E::from_float(L > 0.f ? A / L : 0.f);
}

}  // namespace loki
