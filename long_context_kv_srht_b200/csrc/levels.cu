// levels.cu -- magnitude levels of the RSQ codes (host code).
//
// "Technical Summary: ParisKV", Core Algorithmic Innovations 2, "Quantization": each code is
// one sign bit and a 3-bit magnitude "derived from rotation-induced Beta priors". The codes
// quantise, per 8-dim subspace of the rotated key, r_j = |y_j| / max_i |y_i|. After the
// random rotation a subspace direction is uniform on the sphere (u_j^2 ~ Beta(1/2, 7/2)), so
// u = g / |g| for i.i.d. standard normal g, and r_j = |g_j| / max_i |g_i| does not depend on
// |g|. With psi(t) = sqrt(2/pi) exp(-t^2/2) and Psi(t) = erf(t / sqrt 2) (the half-normal
// density and CDF), r has mass 1/8 at 1 (the maximal coordinate itself) and on [0, 1) the
// density
//     f(x) = 7 * integral_0^inf psi(t) psi(x t) t Psi(t)^6 dt.
// PARISKV_LEVELS_PRIOR uses the 8-level Lloyd-Max quantiser of that law: levels are the
// conditional means of their cells, cells split at the midpoints between levels. They are
// computed here once per process: f by the midpoint rule in t on [0, 9] (the integrand is
// below 1e-17 beyond), cell masses and first moments from cumulative trapezoid integrals of
// f on a uniform grid in x, interpolated at the cell edges, and Lloyd iterations from
// uniform cell midpoints until the levels stop moving.
#include <cmath>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "internal.hpp"

namespace pkv {

namespace {

constexpr int kNx = 8192;       // x grid cells on [0, 1]
constexpr int kNt = 2048;       // t midpoints on [0, kTmax]
constexpr double kTmax = 9.0;
constexpr int kIters = 4000;

std::once_flag g_prior_once;
float g_prior[8];

double interp(const std::vector<double>& F, double x) {
    const double pos = x * kNx;
    int i = static_cast<int>(pos);
    if (i >= kNx) return F[kNx];
    if (i < 0) return F[0];
    const double w = pos - i;
    return F[i] + w * (F[i + 1] - F[i]);
}

void compute_prior() {
    const double c = std::sqrt(2.0 / M_PI);
    const double ht = kTmax / kNt;
    std::vector<double> t(kNt), wt(kNt);
    for (int j = 0; j < kNt; ++j) {
        t[j] = (j + 0.5) * ht;
        const double psi = c * std::exp(-0.5 * t[j] * t[j]);
        const double Psi = std::erf(t[j] / std::sqrt(2.0));
        const double p2 = Psi * Psi;
        wt[j] = psi * t[j] * p2 * p2 * p2 * ht;          // psi(t) t Psi(t)^6 dt
    }
    std::vector<double> F0(kNx + 1, 0.0), F1(kNx + 1, 0.0), f(kNx + 1);
    for (int i = 0; i <= kNx; ++i) {
        const double x = static_cast<double>(i) / kNx;
        double s = 0.0;
        for (int j = 0; j < kNt; ++j) {
            const double xt = x * t[j];
            s += wt[j] * c * std::exp(-0.5 * xt * xt);
        }
        f[i] = 7.0 * s;
    }
    const double hx = 1.0 / kNx;
    for (int i = 1; i <= kNx; ++i) {
        const double x0 = static_cast<double>(i - 1) / kNx, x1 = static_cast<double>(i) / kNx;
        F0[i] = F0[i - 1] + 0.5 * hx * (f[i - 1] + f[i]);
        F1[i] = F1[i - 1] + 0.5 * hx * (x0 * f[i - 1] + x1 * f[i]);
    }
    double lv[8];
    for (int i = 0; i < 8; ++i) lv[i] = (i + 0.5) / 8.0;
    for (int it = 0; it < kIters; ++it) {
        double edge[9];
        edge[0] = 0.0;
        edge[8] = 1.0;
        for (int i = 1; i < 8; ++i) edge[i] = 0.5 * (lv[i - 1] + lv[i]);
        double moved = 0.0;
        for (int i = 0; i < 8; ++i) {
            double s0 = interp(F0, edge[i + 1]) - interp(F0, edge[i]);
            double s1 = interp(F1, edge[i + 1]) - interp(F1, edge[i]);
            if (i == 7) {                                  // the mass 1/8 at r = 1
                s0 += 0.125;
                s1 += 0.125;
            }
            const double nl = s0 > 0.0 ? s1 / s0 : lv[i];
            moved = std::fmax(moved, std::fabs(nl - lv[i]));
            lv[i] = nl;
        }
        if (moved < 1e-13) break;
    }
    for (int i = 0; i < 8; ++i) g_prior[i] = static_cast<float>(lv[i]);
}

}  // namespace

void prior_levels(float out[8]) {
    std::call_once(g_prior_once, compute_prior);
    for (int i = 0; i < 8; ++i) out[i] = g_prior[i];
}

pariskv_status level_tables(const pariskv_config* cfg, float tab[kLevelTableFloats]) {
    for (int i = 0; i < kLevelTableFloats; ++i) tab[i] = 0.0f;
    if (cfg->levels == PARISKV_LEVELS_UNIFORM) {
        for (int i = 0; i < 8; ++i) tab[i] = static_cast<float>(i);
        for (int u = 0; u < 16; ++u) tab[16 + u] = static_cast<float>(u - 8);
        return PARISKV_OK;
    }
    float lv[8];
    if (cfg->levels == PARISKV_LEVELS_PRIOR) {
        prior_levels(lv);
    } else if (cfg->levels == PARISKV_LEVELS_TABLE) {
        for (int i = 0; i < 8; ++i) {
            lv[i] = cfg->level_table[i];
            if (!std::isfinite(lv[i]) || (i == 0 ? lv[i] < 0.0f : !(lv[i] > lv[i - 1])))
                return fail(PARISKV_EINVAL, "level_table must be finite with 0 <= c0 < ... < c7");
        }
    } else {
        return fail(PARISKV_EINVAL, "levels=%d unknown", cfg->levels);
    }
    for (int i = 0; i < 8; ++i) tab[i] = lv[i];
    for (int i = 1; i < 8; ++i)   // fp32 rounding of the exact midpoint
        tab[8 + i] = static_cast<float>((static_cast<double>(lv[i - 1]) + lv[i]) * 0.5);
    for (int u = 0; u < 16; ++u) tab[16 + u] = u >= 8 ? lv[u - 8] : -lv[7 - u];
    return PARISKV_OK;
}

}  // namespace pkv

extern "C" pariskv_status pariskv_prior_levels(float* out) {
    if (!out) return pkv::fail(PARISKV_EINVAL, "out is NULL");
    pkv::prior_levels(out);
    return PARISKV_OK;
}
