/*
 * Exhaustive check that rounding w/s to the nearest integer (ties to even)
 * gives the same integer whether the quotient is formed in IEEE fp32 or in
 * IEEE fp64, for every positive finite bf16 weight w and every positive
 * finite fp16 scale s with w/s <= 512.  (In the RTN quantizer |w/s| <= qmax
 * <= 255 always; the sign is symmetric under both division and rint.)
 * The quantize+pack kernel forms the code's quotient in fp32, the oracle in
 * fp64; this program shows the two decisions never differ.
 * Prints the number of pairs checked and the number of mismatches.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

static float bf16(uint16_t b) { uint32_t u = (uint32_t)b << 16; float f; memcpy(&f, &u, 4); return f; }
static double f16(uint16_t h)
{
    int e = (h >> 10) & 31, m = h & 1023;
    return e ? ldexp(1024.0 + m, e - 25) : ldexp((double)m, -24);
}

int main(void)
{
    unsigned long long checked = 0, bad = 0;
    for (uint32_t sb = 1; sb <= 0x7BFF; sb++) {
        double sd = f16((uint16_t)sb);
        float sf = (float)sd;                       /* exact */
        for (uint32_t wb = 1; wb <= 0x7F7F; wb++) {
            float wf = bf16((uint16_t)wb);
            double wd = (double)wf;
            if (wd > 512.0 * sd) break;              /* bf16 patterns increase with value */
            volatile float qf = wf / sf;
            volatile double qd = wd / sd;
            float rf = rintf(qf);
            double rd = rint(qd);
            checked++;
            if ((double)rf != rd) {
                if (bad < 10) printf("mismatch w=0x%04x s=0x%04x %.9g %.17g\n", wb, sb, rf, rd);
                bad++;
            }
        }
    }
    printf("checked %llu mismatches %llu\n", checked, bad);
    return bad != 0;
}
