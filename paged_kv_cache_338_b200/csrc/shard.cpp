// Host planner that splits a decode batch over several GPUs by sequence.
//
// Decode attention of one sequence reads only that sequence's blocks, so the
// sequences of a batch can be spread over devices with no exchange at all;
// what must be balanced is the K/V each device streams, which grows with the
// context length.  Longest-processing-time-first: sequences in decreasing
// length (a stable order, so equal lengths keep their index order), each to
// the device with the fewest tokens so far (lowest index on ties).
#include <algorithm>
#include <numeric>
#include <vector>

#include "pa_internal.h"

extern "C" pa_status pa_plan_shards(const int32_t* context_lens_host, int S, int ndev,
                                    int32_t* device_of_seq_host, int64_t* tokens_per_device_host) {
    pa::clear_error();
    if (S < 0 || ndev < 1) return pa::fail(PA_ERR_INVALID_ARG, "S must be >= 0 and ndev >= 1");
    if (S > 0 && (!context_lens_host || !device_of_seq_host))
        return pa::fail(PA_ERR_INVALID_ARG, "NULL pointer");
    for (int s = 0; s < S; ++s)
        if (context_lens_host[s] < 0)
            return pa::fail(PA_ERR_INVALID_ARG, "context_lens[%d] = %d < 0", s, context_lens_host[s]);
    std::vector<int> order(S);
    std::iota(order.begin(), order.end(), 0);
    std::stable_sort(order.begin(), order.end(), [&](int a, int b) {
        return context_lens_host[a] > context_lens_host[b];
    });
    std::vector<int64_t> load(ndev, 0);
    for (int s : order) {
        const int d = (int)(std::min_element(load.begin(), load.end()) - load.begin());
        device_of_seq_host[s] = d;
        load[d] += context_lens_host[s];
    }
    if (tokens_per_device_host) std::copy(load.begin(), load.end(), tokens_per_device_host);
    return PA_OK;
}
