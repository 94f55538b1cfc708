#pragma once
#include "mala_ptx.cuh"
