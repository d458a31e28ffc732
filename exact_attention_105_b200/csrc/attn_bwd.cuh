#pragma once
#include "sm100.cuh"
