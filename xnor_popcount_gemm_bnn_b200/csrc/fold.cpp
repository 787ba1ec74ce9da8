// Host-side fold of inference BatchNorm + sign into an integer popcount
// threshold per output channel.
//
// "Binary Neural Network (BNN)" glossary, BatchNorm paragraph: BatchNorm
// normalises the (alpha-scaled) output of a binary layer before it is
// binarised again for the next layer.  The pages give no formula; the
// decision folded here is standard inference BatchNorm of alpha*s followed by
// the sign rule of "Extreme Quantization: Binary, Ternary & 1-bit LLMs"
// (Notation: >= 0 -> +1), evaluated in IEEE double in this order:
//
//     v(s) = ((alpha*s - mean) / sqrt(var + eps)) * gamma + beta,   +1 iff v >= 0.
//
// With alpha >= 0 and sqrt(var + eps) > 0, every step is monotone in s
// (correctly rounded multiply, subtract, divide and add are monotone), so
// the set {s : v(s) >= 0} is an up-set when gamma > 0 and a down-set when
// gamma < 0.  Over the reachable s = K - 2d (d = popcount of the XOR, 0..K)
// the decision is therefore a single threshold on d, found here by binary
// search with the same expression -- exact for every d by construction.
// Compiled without floating-point contraction so that no fused multiply-add
// changes the rounding of the expression above.
#include <cmath>
#include <cstdint>

#include "bnn.h"

namespace {

inline bool bn_positive(double a, double g, double b, double mu, double denom, int64_t K, int64_t d) {
    const double s = (double)(K - 2 * d);
    const double x = a * s;
    const double v = (x - mu) / denom * g + b;
    return v >= 0.0;
}

}  // namespace

extern "C" bnn_status bnn_fold_bn_threshold(const float* alpha, const float* gamma, const float* beta,
                                            const float* mean, const float* var, double eps, int64_t N,
                                            int64_t K, int32_t* popc_thresh, int8_t* thresh_mode) {
    if (N < 0 || K < 1 || K > INT32_MAX / 2) return BNN_ERR_INVALID_ARG;
    if (N == 0) return BNN_OK;
    if (!alpha || !gamma || !beta || !mean || !var || !popc_thresh || !thresh_mode)
        return BNN_ERR_INVALID_ARG;
    if (!std::isfinite(eps)) return BNN_ERR_INVALID_ARG;
    for (int64_t n = 0; n < N; ++n) {
        const double a = alpha[n], g = gamma[n], b = beta[n], mu = mean[n], v = var[n];
        if (!std::isfinite(a) || !std::isfinite(g) || !std::isfinite(b) || !std::isfinite(mu) ||
            !std::isfinite(v) || a < 0.0)
            return BNN_ERR_INVALID_ARG;
        const double ve = v + eps;
        if (!(ve > 0.0)) return BNN_ERR_INVALID_ARG;
    }
    for (int64_t n = 0; n < N; ++n) {
        const double a = alpha[n], g = gamma[n], b = beta[n], mu = mean[n];
        const double denom = std::sqrt((double)var[n] + eps);
        const bool pos0 = bn_positive(a, g, b, mu, denom, K, 0);   // s = +K
        const bool posK = bn_positive(a, g, b, mu, denom, K, K);   // s = -K
        if (pos0 == posK) {
            // Monotone with equal end points: the decision is constant.
            thresh_mode[n] = 0;
            popc_thresh[n] = pos0 ? (int32_t)K : -1;
        } else if (pos0) {
            // +1 for small d (gamma > 0): largest d with v >= 0; bit = (d > D).
            int64_t lo = 0, hi = K;          // pos(lo) true, pos(hi) false
            while (hi - lo > 1) {
                const int64_t mid = lo + (hi - lo) / 2;
                if (bn_positive(a, g, b, mu, denom, K, mid)) lo = mid; else hi = mid;
            }
            thresh_mode[n] = 0;
            popc_thresh[n] = (int32_t)lo;
        } else {
            // +1 for large d (gamma < 0): smallest d with v >= 0; bit = (d < D).
            int64_t lo = 0, hi = K;          // pos(lo) false, pos(hi) true
            while (hi - lo > 1) {
                const int64_t mid = lo + (hi - lo) / 2;
                if (bn_positive(a, g, b, mu, denom, K, mid)) hi = mid; else lo = mid;
            }
            thresh_mode[n] = 1;
            popc_thresh[n] = (int32_t)hi;
        }
    }
    return BNN_OK;
}
