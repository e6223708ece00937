// phi(q) and phi(k) written once to scratch before the tensor-core prefill.
//
// With a feature map other than the identity (page "MiniMax-M1で理解する…",
// section "線形アテンションの数学的基礎": phi(Q) (phi(K)^T V)), the prefill reads
// phi(Q) and phi(K) as tensor-core operands in bf16.  For elu + 1, mapping
// them in a separate bandwidth-bound pass (read 2, write 2 arrays) costs less
// than evaluating the exponentials on the tiles inside the pipelined kernel,
// where the mapping sits on the chain that feeds the next chunk's product
// (relu, one packed max per pair, is cheaper inside).  Both use
// apply_phi_bf16x8, so the two routes give bit-identical operands.
#pragma once
#include "phi.cuh"

namespace lcl {
namespace phimap {

constexpr int NUM_THREADS = 256;
constexpr int VPT = 4;  // 16-byte vectors in flight per thread

// a, b: n vectors of 8 bf16 each; ya = phi(a), yb = phi(b).
__global__ void __launch_bounds__(NUM_THREADS)
phi_map_kernel(const uint4* __restrict__ a, const uint4* __restrict__ b, uint4* __restrict__ ya,
               uint4* __restrict__ yb, long n, int phi) {
    const long total = 2 * n;
    const long step = (long)gridDim.x * NUM_THREADS * VPT;
    for (long base = (long)blockIdx.x * NUM_THREADS * VPT + threadIdx.x; base < total; base += step) {
        uint4 r[VPT];
#pragma unroll
        for (int j = 0; j < VPT; ++j) {
            const long e = base + (long)j * NUM_THREADS;
            if (e < total) r[j] = e < n ? a[e] : b[e - n];
        }
#pragma unroll
        for (int j = 0; j < VPT; ++j) {
            const long e = base + (long)j * NUM_THREADS;
            if (e < total) {
                const uint4 y = apply_phi_bf16x8(r[j], phi);
                if (e < n) ya[e] = y;
                else yb[e - n] = y;
            }
        }
    }
}

}  // namespace phimap
}  // namespace lcl
