// Host-side builder of the minimal symmetric basis M_p and multiplicities C_p.
//
// [CC-TAYLOR] = "Self-attention at constant cost per token via symmetry-aware
// Taylor approximation" (blog.hotdry.top).  Section "The Taylor approximation"
// (泰勒近似的数学突破): (q.k)^p is a sum over the symmetric tensors q^{(x)p},
// k^{(x)p}; keeping one representative per monomial (the upper-triangular
// tuples) leaves binom(d_K+p-1, p) coordinates.  Section "Feature maps and
// linear attention" (特征映射与线性注意力): C_p holds how often each monomial
// occurs in the full expansion.  Section "Hardware optimization paths"
// (硬件优化实现路径): rows of M_p are nondecreasing, i1 <= ... <= ip.
//
// Order: degrees p = 0..P-1 concatenated; within a degree, lexicographic.
#include <cstdint>
#include <vector>

#include "sata_internal.h"

namespace sata {

namespace {

// Append every nondecreasing tuple of length p over [lo, d) to `out`, in
// lexicographic order, by fixing the leading index and recursing on the rest.
void append_tuples(int d, int p, int lo, std::vector<uint8_t> &prefix,
                   std::vector<std::vector<uint8_t>> &out) {
    if ((int)prefix.size() == p) {
        out.push_back(prefix);
        return;
    }
    for (int i = lo; i < d; ++i) {
        prefix.push_back((uint8_t)i);
        append_tuples(d, p, i, prefix, out);
        prefix.pop_back();
    }
}

uint64_t fact(int n) {
    uint64_t r = 1;
    for (int i = 2; i <= n; ++i) r *= (uint64_t)i;
    return r;
}

}  // namespace

int64_t binom64(int n, int k) {
    if (k < 0 || n < 0 || k > n) return 0;
    int64_t r = 1;
    for (int i = 1; i <= k; ++i) r = r * (n - k + i) / i;
    return r;
}

int64_t num_features(int d_K, int P) { return binom64(d_K + P - 1, P - 1); }

bool build_basis_host(int d_K, int P, HostBasis &hb) {
    if (d_K < 1 || d_K > 255 || P < 1 || P > kMaxP + 4) return false;
    hb.d_K = d_K;
    hb.P = P;
    hb.tuples.clear();
    hb.degree.clear();
    hb.mult.clear();
    hb.offsets.assign(P + 1, 0);
    for (int p = 0; p < P; ++p) {
        hb.offsets[p] = (int64_t)hb.tuples.size();
        std::vector<std::vector<uint8_t>> tup;
        std::vector<uint8_t> prefix;
        append_tuples(d_K, p, 0, prefix, tup);
        for (auto &t : tup) {
            // multiplicity = p! / prod over runs of equal indices of (run length)!
            uint64_t c = fact(p);
            size_t s = 0;
            while (s < t.size()) {
                size_t e = s;
                while (e < t.size() && t[e] == t[s]) ++e;
                c /= fact((int)(e - s));
                s = e;
            }
            hb.tuples.push_back(t);
            hb.degree.push_back((uint8_t)p);
            hb.mult.push_back((uint32_t)c);
        }
    }
    hb.offsets[P] = (int64_t)hb.tuples.size();
    return hb.offsets[P] == num_features(d_K, P);
}

}  // namespace sata
