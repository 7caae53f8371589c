/* Driver of the threaded race check (tests/test_simt_host_threads.py): runs the
 * CUDA-core kernels -- one-pass forward, momentum, the two-pass form's first
 * and second passes, the states-only forward and the backward -- on a small
 * request (two value heads, a ragged last chunk, two value tiles), one host
 * thread per CUDA thread, 256 per CTA, CTAs one after another.  argv: G, then
 * the inverse (0 exact, 1 truncated Neumann with two Newton steps, 2 1-Step
 * Neumann).  The kernels' source is prepended by the test. */
#include <cstdio>
#include <random>
#include <thread>
#include <vector>
thread_local host_uint3 threadIdx, blockIdx, gridDim;
std::barrier<> *host_cta_barrier;
static std::vector<float> g_smem(227 * 1024 / 4);
float *host_smem_ptr() { return g_smem.data(); }

template <class F>
static void run_cta(unsigned x, unsigned y, unsigned z, F &&body)
{
    std::barrier<> bar(256);
    host_cta_barrier = &bar;
    std::fill(g_smem.begin(), g_smem.end(), std::nanf(""));
    std::vector<std::thread> th;
    for (unsigned t = 0; t < 256; ++t)
        th.emplace_back([&, t] { threadIdx = {t, 0, 0}; blockIdx = {x, y, z}; body(); });
    for (auto &h : th) h.join();
}

int main(int argc, char **argv)
{
    // a small request with every feature in play: grouped values, ragged last chunk
    const int B = 1, T = 21, Hk = 1, Hv = 2, dk = 16, dv = 40, C = 8;
    const int G = argc > 1 ? atoi(argv[1]) : 16;
    const int inv = argc > 2 ? atoi(argv[2]) : 0;   // 0 exact, 1 neumann, 2 neumann1
    std::mt19937 rng(7);
    std::normal_distribution<float> N(0.f, 1.f);
    auto vec = [&](size_t n, float s) { std::vector<float> a(n); for (auto &x : a) x = s * N(rng); return a; };
    auto q = vec((size_t)B * Hk * T * dk, 0.25f), k = vec((size_t)B * Hk * T * dk, 0.25f);
    auto v = vec((size_t)B * Hv * T * dv, 1.f), S0 = vec((size_t)B * Hv * dk * dv, 0.5f);
    auto g = vec((size_t)B * Hk * T * G, 0.3f), beta = vec((size_t)B * Hk * T, 1.f);
    for (auto &x : g) x = -std::log1p(std::exp(x));
    for (auto &x : beta) x = 1.f / (1.f + std::exp(-x));
    const int nch = (T + C - 1) / C;
    std::vector<float> o((size_t)B * Hv * T * dv), Sf((size_t)B * Hv * dk * dv), o2(o.size()), Sf2(Sf.size());
    std::vector<float> rec((size_t)B * Hk * nch * 2 * C * C, std::nanf(""));
    std::vector<float> Sc((size_t)B * Hv * nch * dk * dv);
    gdr::Params p{};
    p.B = B; p.T = T; p.Hk = Hk; p.Hv = Hv; p.dk = dk; p.dv = dv; p.G = G; p.C = C; p.R = Hv / Hk;
    p.neumann = inv == 1; p.neumann1 = inv == 2; p.neu_order = inv == 1 ? 3 : 0; p.neu_resid = inv == 1 ? 2 : 0;
    p.q = q.data(); p.k = k.data(); p.v = v.data(); p.g = g.data(); p.beta = beta.data(); p.S0 = S0.data();
    p.o = o.data(); p.S_final = Sf.data();
    const int ntile = (dv + 31) / 32;
    // one-pass forward
    for (int b = 0; b < B; ++b) for (int h = 0; h < Hv; ++h) for (int x = 0; x < ntile; ++x)
        run_cta(x, h, b, [&] { gdr::emu_f::simt_fwd_kernel<false, false, 32, false, false>(p); });
    // momentum
    gdr::Params pm = p; pm.momentum = 1; pm.mu = 0.5f; pm.o = o2.data(); pm.S_final = Sf2.data();
    for (int b = 0; b < B; ++b) for (int h = 0; h < Hv; ++h) for (int x = 0; x < ntile; ++x)
        run_cta(x, h, b, [&] { gdr::emu_f::simt_fwd_kernel<false, false, 32, true, false>(pm); });
    // two-pass: factors, then the value tiles reading them
    for (int b = 0; b < B; ++b) for (int h = 0; h < Hk; ++h) for (int c = 0; c < nch; ++c)
        run_cta(c, h, b, [&] { gdr::emu_f::simt_factors_kernel<false>(p, rec.data()); });
    gdr::Params p2 = p; p2.factors = rec.data(); p2.o = o2.data(); p2.S_final = Sf2.data();
    for (int b = 0; b < B; ++b) for (int h = 0; h < Hv; ++h) for (int x = 0; x < ntile; ++x)
        run_cta(x, h, b, [&] { gdr::emu_f::simt_fwd_kernel<false, false, 32, false, true>(p2); });
    double d2 = 0, m2 = 0;
    for (size_t i = 0; i < o.size(); ++i) { d2 = std::max(d2, (double)std::fabs(o[i] - o2[i])); m2 = std::max(m2, (double)std::fabs(o[i])); }
    printf("two-pass vs one-pass: max|do| / max|o| = %.2e\n", d2 / m2);
    if (inv == 0) {   // backward: states-only forward, then the reverse sweep
        gdr::Params pf = p; pf.o = nullptr; pf.S_final = nullptr; pf.S_chunks = Sc.data();
        for (int b = 0; b < B; ++b) for (int h = 0; h < Hv; ++h) for (int x = 0; x < ntile; ++x)
            run_cta(x, h, b, [&] { gdr::emu_f::simt_fwd_kernel<false, false, 32, false, false>(pf); });
        auto dO = vec(o.size(), 1.f), dSf = vec(Sf.size(), 1.f);
        std::vector<float> gq(q.size()), gk(k.size()), gv(v.size()), gg(g.size()), gb(beta.size()), gS(S0.size());
        gdr::Params pb = p; pb.S_chunks = Sc.data(); pb.dO = dO.data(); pb.dS_final = dSf.data();
        pb.grad_q = gq.data(); pb.grad_k = gk.data(); pb.grad_v = gv.data(); pb.grad_g = gg.data();
        pb.grad_beta = gb.data(); pb.grad_S0 = gS.data();
        for (int b = 0; b < B; ++b) for (int h = 0; h < Hv; ++h) for (int x = 0; x < ntile; ++x)
            run_cta(x, h, b, [&] { gdr::emu_b::simt_bwd_kernel<false, 32>(pb); });
        double s = 0; for (float x : gq) s += x; printf("backward ran, sum dq = %.4f\n", s);
    }
    printf("done G=%d inverse=%d\n", G, inv);
    return 0;
}
