// Single translation unit of the KDA CUDA library (sm_100a).  The parts are
// kept in separate files by concern and compiled together so that the
// per-device status word needs no relocatable device code.
#include "kda_api.cu"
#include "kda_decode.cu"
#include "kda_chunk_simt.cu"
#include "kda_chunk_split.cu"
#include "kda_chunk_bwd.cu"
#include "kda_dplr.cu"
