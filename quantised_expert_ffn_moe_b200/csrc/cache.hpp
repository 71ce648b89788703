// cache.hpp -- expert residency cache (host policy): which of a bounded set of
// slots holds each expert a token routes to, and which experts must be copied
// in.  Pages: "Flash-MoE - Exécuter un modèle de 397 milliards de paramètres
// sur un ordinateur portable", "SSD Expert Streaming" (only the active experts
// are brought in, per token); "104 Go de modèle sur un Mac de 48 Go" (a fixed
// number of expert slots); consecutive tokens reuse some experts.
//
// Policy: an expert already resident is a hit and keeps its slot; a miss takes
// the lowest-numbered empty slot, else the least recently used slot that the
// current token does not need (ties to the lower slot).  Deterministic.
#pragma once

#include <cstdint>
#include <vector>

namespace moeq {

class ExpertCache {
public:
    ExpertCache(int n_experts, int n_slots)
        : n_experts_(n_experts), n_slots_(n_slots), slot_of_(n_experts, -1), expert_in_(n_slots, -1),
          last_use_(n_slots, 0), seen_(n_experts, 0) {}

    int n_experts() const { return n_experts_; }
    int n_slots() const { return n_slots_; }
    int64_t hits() const { return hits_; }
    int64_t misses() const { return misses_; }

    // Returns 0, or -1 for an id out of range or repeated (nothing changed).
    int plan(const int32_t *ids, int k, int32_t *slot_of, int32_t *fill_ids, int32_t *fill_slots, int32_t *n_fill) {
        ++tick_;
        for (int i = 0; i < k; ++i) {
            const int e = ids[i];
            if (e < 0 || e >= n_experts_ || seen_[e] == tick_) return -1;
            seen_[e] = tick_;
        }
        // hits first: their slots count as used by this token
        for (int i = 0; i < k; ++i) {
            const int s = slot_of_[ids[i]];
            if (s >= 0) last_use_[s] = tick_;
        }
        int nf = 0;
        for (int i = 0; i < k; ++i) {
            const int e = ids[i];
            int s = slot_of_[e];
            if (s >= 0) {
                ++hits_;
            } else {
                ++misses_;
                s = victim();
                if (expert_in_[s] >= 0) slot_of_[expert_in_[s]] = -1;
                expert_in_[s] = e;
                slot_of_[e] = s;
                last_use_[s] = tick_;
                fill_ids[nf] = e;
                fill_slots[nf] = s;
                ++nf;
            }
            slot_of[i] = s;
        }
        *n_fill = nf;
        return 0;
    }

private:
    // The slot a miss refills: an empty one (lowest index), else the least
    // recently used one not used by this token (lowest index on ties).
    int victim() const {
        int best = -1;
        for (int s = 0; s < n_slots_; ++s) {
            if (expert_in_[s] < 0) return s;
            if (last_use_[s] == tick_) continue;
            if (best < 0 || last_use_[s] < last_use_[best]) best = s;
        }
        return best;  // exists: k <= n_slots, so some slot is free of this token
    }

    int n_experts_, n_slots_;
    std::vector<int> slot_of_;       // expert -> slot, or -1
    std::vector<int> expert_in_;     // slot -> expert, or -1
    std::vector<uint64_t> last_use_; // slot -> tick of last use
    std::vector<uint64_t> seen_;     // expert -> tick of the last plan that listed it
    uint64_t tick_ = 0;
    int64_t hits_ = 0, misses_ = 0;
};

}  // namespace moeq
