#pragma once
#include "fa_ptx.cuh"
