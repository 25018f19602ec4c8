// Fastest forward path per (I/O dtype, channels B*C, tokens T), measured on NVIDIA B200
// by linear_attention_rnn_wkv_b200/tune.py on 2026-12-03 (CUDA-event
// timings of back-to-back launches on inputs larger than the L2).  Entries: 1 the serial
// path, 8 or 16 the chunked path with that chunk length; 0 a point not measured (too
// large), which takes its nearest measured neighbour in T.  Regenerate with the tuning
// script and rebuild the library.
#pragma once

namespace wkvb {

constexpr int kTuneNumBC = 6;
constexpr int kTuneNumT = 8;
constexpr long long kTuneBC[kTuneNumBC] = {64, 512, 4096, 32768, 262144, 1048576};
constexpr long long kTuneT[kTuneNumT] = {1, 4, 16, 64, 256, 1024, 4096, 16384};
// [dtype: 0 fp32, 1 bf16][B*C][T]
constexpr signed char kTunePath[2][kTuneNumBC][kTuneNumT] = {
    {
        {1, 1, 1, 8, 8, 16, 16, 16},  // B*C = 64
        {1, 1, 1, 8, 8, 8, 16, 16},  // B*C = 512
        {1, 1, 1, 16, 16, 16, 16, 16},  // B*C = 4096
        {1, 1, 1, 8, 16, 16, 16, 0},  // B*C = 32768
        {1, 1, 8, 8, 16, 16, 0, 0},  // B*C = 262144
        {1, 1, 8, 8, 16, 0, 0, 0},  // B*C = 1048576
    },
    {
        {1, 1, 1, 8, 16, 16, 16, 16},  // B*C = 64
        {1, 1, 1, 8, 16, 16, 16, 16},  // B*C = 512
        {1, 1, 1, 8, 16, 16, 16, 16},  // B*C = 4096
        {1, 1, 1, 8, 16, 16, 16, 0},  // B*C = 32768
        {1, 1, 1, 8, 16, 16, 0, 0},  // B*C = 262144
        {1, 1, 1, 8, 16, 0, 0, 0},  // B*C = 1048576
    },
};

}  // namespace wkvb
