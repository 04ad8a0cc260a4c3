// cq_codebook.cpp -- host-side default codebooks for libcq (setup, not the data path).
//
// Page "How Quantization Codebooks Are Trained in Cactus Quants":
//   * samples: NumPy-legacy RandomState(seed).randn(400000), i.e. MT19937 seeded with the
//     reference init_genrand recurrence (std::mt19937 implements exactly that engine),
//     53-bit doubles from two 32-bit draws, Marsaglia's polar method returning the cached
//     second deviate of each accepted pair ("Gaussian Sampling and Initialization");
//   * 1-D Lloyd-Max: quantile initialisation, then 200 rounds of midpoint boundaries,
//     left-sided searchsorted assignment and cell means; result sorted ("Iterative
//     Refinement of Quantization Levels");
//   * ternary: the hard-coded three levels ("Ternary Special Case Handling");
//   * scale by 1/sqrt(group_size), memoised per arguments ("Production Codebook Generation
//     and Caching").
// Because the samples are sorted, every cell is a contiguous run: boundaries are found by
// binary search and each cell's sum is taken over its run in ascending order.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <map>
#include <mutex>
#include <random>
#include <tuple>
#include <vector>

#include "cq_internal.h"

namespace {

// NumPy legacy gauss on top of the standard MT19937 engine.
class LegacyNormal {
  public:
    explicit LegacyNormal(uint32_t seed) : eng_(seed) {}
    double next() {
        if (cached_) {
            cached_ = false;
            return spare_;
        }
        double a, b, s;
        do {
            a = 2.0 * uniform53() - 1.0;
            b = 2.0 * uniform53() - 1.0;
            s = a * a + b * b;
        } while (s >= 1.0 || s == 0.0);
        const double f = std::sqrt(-2.0 * std::log(s) / s);
        spare_ = f * a;
        cached_ = true;
        return f * b;
    }

  private:
    double uniform53() {
        const uint32_t hi = static_cast<uint32_t>(eng_()) >> 5;
        const uint32_t lo = static_cast<uint32_t>(eng_()) >> 6;
        return (hi * 67108864.0 + lo) / 9007199254740992.0;
    }
    std::mt19937 eng_;
    bool cached_ = false;
    double spare_ = 0.0;
};

std::vector<double> lloyd_max(int levels, int samples, int iters, uint32_t seed) {
    std::vector<double> x(samples);
    LegacyNormal gen(seed);
    for (auto& v : x) v = gen.next();
    std::sort(x.begin(), x.end());

    std::vector<double> c(levels);
    for (int k = 0; k < levels; ++k)
        c[k] = x[static_cast<size_t>((k + 0.5) / levels * samples)];

    std::vector<size_t> edge(levels + 1);
    for (int it = 0; it < iters; ++it) {
        // cell k = (b_{k-1}, b_k]: the samples a left-sided searchsorted assigns to k
        edge[0] = 0;
        edge[levels] = x.size();
        for (int k = 0; k + 1 < levels; ++k) {
            const double b = (c[k] + c[k + 1]) / 2.0;
            edge[k + 1] = std::upper_bound(x.begin(), x.end(), b) - x.begin();
        }
        for (int k = 0; k < levels; ++k) {
            const size_t lo = edge[k], hi = std::max(edge[k], edge[k + 1]);
            if (hi <= lo) continue;  // empty cell keeps its level
            double s = 0.0;
            for (size_t i = lo; i < hi; ++i) s += x[i];
            c[k] = s / static_cast<double>(hi - lo);
        }
    }
    std::sort(c.begin(), c.end());
    return c;
}

std::mutex g_mu;
std::map<std::tuple<int, int, unsigned long long>, std::vector<float>> g_memo;

}  // namespace

namespace cq {

int levels_for_bits(int bits) {
    if (bits == CQ_BITS_TERNARY) return 3;
    if (bits >= 2 && bits <= 4) return 1 << bits;
    return -1;
}

int field_bits_for(int bits) {
    if (bits == CQ_BITS_TERNARY) return 2;
    if (bits >= 2 && bits <= 4) return bits;
    return -1;
}

int host_codebook(int bits, int group_size, unsigned long long seed, float* out) {
    const int L = levels_for_bits(bits);
    if (L < 0 || group_size < 8 || group_size > 4096 || (group_size & (group_size - 1)))
        return -1;
    if (bits == CQ_BITS_TERNARY) seed = 0;
    const auto key = std::make_tuple(bits, group_size, seed);
    std::lock_guard<std::mutex> lock(g_mu);
    auto it = g_memo.find(key);
    if (it == g_memo.end()) {
        std::vector<double> lv;
        if (bits == CQ_BITS_TERNARY)
            lv = {-1.2240064, 0.0, 1.2240064};
        else
            lv = lloyd_max(L, 400000, 200, static_cast<uint32_t>(seed));
        const double s = std::sqrt(static_cast<double>(group_size));
        std::vector<float> cb(L);
        for (int k = 0; k < L; ++k) cb[k] = static_cast<float>(lv[k] / s);
        it = g_memo.emplace(key, std::move(cb)).first;
    }
    std::copy(it->second.begin(), it->second.end(), out);
    return L;
}

}  // namespace cq
