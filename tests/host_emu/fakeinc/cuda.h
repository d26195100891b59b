#pragma once
struct alignas(64) CUtensorMap { unsigned long long opaque[16]; };
