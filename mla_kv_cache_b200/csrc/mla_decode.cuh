// mla_decode.cuh -- absorbed-MLA decode (latent 512 + RoPE 64).
#pragma once
#include "common.cuh"
