// Prints the library's host E4M3 encoding of the float32 bit patterns read from stdin (one
// hexadecimal pattern per line), one two-digit hexadecimal code per line; the test compares
// them with an encoding written from the format's definition.
#include <cstdint>
#include <cstdio>
#include <cstring>

#include "e4m3.h"

int main() {
    unsigned u;
    while (std::scanf("%x", &u) == 1) {
        float f;
        std::memcpy(&f, &u, 4);
        std::printf("%02x\n", jd::e4m3_encode(f));
    }
    return 0;
}
