// Host-built constant tables of the E8 core (library side).
//
// The core is the set of 65,536 E8 points that come first when the points
// are ordered by |p|^2 and then lexicographically by doubled coordinates
// P = 2p (most negative first); a core index is the rank in that order
// (E8-QAT appendix Table 3: 65,536 core codewords).  Points are handled in
// doubled coordinates: all P_i even or all odd, sum(P) divisible by 4.
//
// Ranking without a search: split P into a head H = (P0..P3) and a tail
// L = (P4..P7), each coordinate mapped to a digit (P_i + 6) >> 1 in 0..6,
// key = base-7 number of the four digits.  For points of one type (even or
// odd coordinates) the rank decomposes as
//     rank(P) = T1[type][key(H)][|P|^2 / 8] + T2[type][key(L)],
// where T2 is the lexicographic position of L among the 4-vectors of its
// own type with the same |L|^2 and the same sum mod 4, and T1 absorbs
// everything that only depends on H and |P|^2 (the points of smaller norm,
// the points of the other type whose first coordinate is smaller, and the
// same-type points with a lexicographically smaller head).  T1 is stored
// saturated at 0xFFFF: that value, or T1 + T2 >= 65536, means "not in the
// core".  The builder checks the decomposition on every point.
#pragma once
#include <cstdint>
#include <vector>

namespace e8q {

constexpr int kCoreSize = 65536;
constexpr int kNumRoots = 240;
constexpr int kKeySpace = 2401;              // 7^4 head / tail keys
constexpr int kNormLevels = 7;               // |P|^2 / 8 in 0..6 (|p|^2 <= 12)
constexpr int kT1Size = 2 * kKeySpace * kNormLevels;
constexpr int kT2Size = 2 * kKeySpace;

// Extended set: every E8 point with |p|^2 <= 22 (|P|^2 <= 88), ranked the
// same way (|p|^2, then lexicographic on P); its first 65,536 points are the
// core.  No point outside it can be an escape: |p|^2 >= 24 gives
// |p - r|^2 >= (sqrt(24) - sqrt(2))^2 > 12 for every root r.  Digits
// (P_i + 9) >> 1 in 0..9 (|P_i| <= 9), keys base 10, and the same two-table
// rank: ext_rank(P) = T1e[type][key(H)][|P|^2 / 8] + T2e[type][key(L)].
constexpr int kExtKeySpace = 10000;
constexpr int kExtNormLevels = 12;  // |P|^2 / 8 in 0..11
constexpr int kExtMaxN2 = 88;
constexpr int kExtT1Size = 2 * kExtKeySpace * kExtNormLevels;
constexpr int kExtT2Size = 2 * kExtKeySpace;
constexpr uint32_t kExtNone = 0xFFFFFFFFu;

struct HostTables {
    std::vector<uint16_t> t1;     // [2][2401][7]
    std::vector<uint16_t> t2;     // [2][2401]
    std::vector<int8_t> core;     // [65536][8] doubled coordinates
    std::vector<int8_t> roots;    // [240][8]
    std::vector<uint8_t> root_of_key;  // [512] root index by construction key (see root_key)
    std::vector<uint32_t> t1e;    // [2][10000][12], kExtNone where no point
    std::vector<uint32_t> t2e;    // [2][10000]
    // Encoding of every extended point, by extended rank: k for a core point;
    // rank(p - r) | (root index << 16) | (1 << 24) for an escape (r the root
    // of the escape rule); 2 << 24 when p - r is outside the core.
    std::vector<uint32_t> res;
    bool ok = false;
};

// Extended rank of a doubled E8 point, or kExtNone outside the extended set.
uint32_t ext_rank(const HostTables& t, const int (&P)[8]);

// Root construction key: +-2 at positions i < j (signs si, sj, 1 = minus):
// (i << 5) | (j << 2) | (si << 1) | sj; +-1 everywhere with minus mask m:
// 256 | m.
// Builds the tables once (thread-safe); returns nullptr if a consistency
// check failed.
const HostTables* host_tables();

}  // namespace e8q
