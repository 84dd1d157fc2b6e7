// Calibration side path, step 2: the head-shared angle phi*_k in closed form.
//
// "When Local Variance Optimality Is Not Enough: RoPE-Aligned Q/K Rotations for
// Dynamic 4-Bit Quantisation", "Optimisation objective": for one angle shared by all
// heads of a layer per frequency pair, the angle that minimises the larger channel
// variance under the pooled-covariance, position-averaged surrogate.  With
// y1 = a cos(phi) - b sin(phi), y2 = a sin(phi) + b cos(phi) and covariance
// [[A, C], [C, D]]:
//   max(Var y1, Var y2) = (A + D)/2 + |((A - D)/2) cos 2phi - C sin 2phi| >= (A + D)/2,
// with equality at phi* = atan2(A - D, 2C) / 2 (mod pi/2).  "Estimation strategies"
// gives the three covariances (pooled raw accumulators then centred; K only; equal
// weights on the Q and K uncentred moments, then centred).  fp64 throughout; one
// thread per pair.  A stream the estimator needs with no observations leaves the pair at
// phi = 0 and sets QKQ_STATUS_EMPTY_STREAM.
#include <cuda_runtime.h>
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace qkq {

namespace {

__global__ void k_solve_angles(const double *__restrict__ m, int P, int estimator,
                               float *__restrict__ phi, double *__restrict__ min_maxvar,
                               int *__restrict__ status)
{
    wait_prior_grid();  // the moments are the previous kernel's output
    const int k = blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= P) return;
    const double *q = m + static_cast<size_t>(k) * 6;            // stream 0 (Q)
    const double *kk = m + static_cast<size_t>(P + k) * 6;       // stream 1 (K)
    // a stream the estimator uses without observations (n = 0) has no covariance: the pair
    // keeps the identity rotation (phi = 0) and the call reports it
    const bool empty = estimator == 0   ? !(q[0] + kk[0] > 0.0)
                       : estimator == 1 ? !(kk[0] > 0.0)
                                        : !(q[0] > 0.0 && kk[0] > 0.0);
    if (empty) {
        phi[k] = 0.0f;
        if (min_maxvar != nullptr) min_maxvar[k] = __longlong_as_double(0x7ff8000000000000ll);
        if (status != nullptr) atomicOr(status, ST_EMPTY_STREAM);
        return;
    }
    double m1a, m1b, m2aa, m2ab, m2bb;
    if (estimator == 0) {          // pooled: add raw accumulators, then normalise
        const double n = q[0] + kk[0];
        m1a = (q[1] + kk[1]) / n;
        m1b = (q[2] + kk[2]) / n;
        m2aa = (q[3] + kk[3]) / n;
        m2ab = (q[4] + kk[4]) / n;
        m2bb = (q[5] + kk[5]) / n;
    } else if (estimator == 1) {   // K only
        const double n = kk[0];
        m1a = kk[1] / n;
        m1b = kk[2] / n;
        m2aa = kk[3] / n;
        m2ab = kk[4] / n;
        m2bb = kk[5] / n;
    } else {                       // balanced: mean of the per-stream normalised moments
        const double nq = q[0], nk = kk[0];
        m1a = 0.5 * (q[1] / nq + kk[1] / nk);
        m1b = 0.5 * (q[2] / nq + kk[2] / nk);
        m2aa = 0.5 * (q[3] / nq + kk[3] / nk);
        m2ab = 0.5 * (q[4] / nq + kk[4] / nk);
        m2bb = 0.5 * (q[5] / nq + kk[5] / nk);
    }
    const double A = m2aa - m1a * m1a;
    const double C = m2ab - m1a * m1b;
    const double D = m2bb - m1b * m1b;
    const double tr = A + D;
    double ph = 0.0;
    const double quarter = 0.78539816339744830962;   // pi/4
    if (tr > 0.0 && fabs(A - D) + 2.0 * fabs(C) > 1e-12 * tr) {
        ph = 0.5 * atan2(A - D, 2.0 * C);
        if (ph <= -quarter)
            ph += 2.0 * quarter;
        else if (ph > quarter)
            ph -= 2.0 * quarter;
    }
    phi[k] = static_cast<float>(ph);
    if (min_maxvar != nullptr) {
        const double c = cos(ph), s = sin(ph);
        const double v1 = A * c * c - 2.0 * C * s * c + D * s * s;
        const double v2 = A * s * s + 2.0 * C * s * c + D * c * c;
        min_maxvar[k] = v1 > v2 ? v1 : v2;
    }
}

}  // namespace

cudaError_t solve_angles_launch(const double *moments, int P, int estimator, float *phi,
                                double *min_maxvar, int *status, cudaStream_t stream)
{
    return launch_after_prior(k_solve_angles, dim3(1), dim3(64), 0, stream, moments, P, estimator,
                              phi, min_maxvar, status);
}

}  // namespace qkq
